"""Thin Python binding of libflux (ctypes): the same names as the C ABI in
include/flux.h, argument marshalling only.

Every function takes torch tensors that already live on the GPU, checks dtype,
device, contiguity and shape, and passes raw pointers, sizes and the current CUDA
stream to the library.  All arithmetic runs in the library's kernels; there is no
CPU fallback: if libflux.so is missing or cannot load, every call raises.

With FLUX_CHECKED=1 in the environment the binding loads libflux_checked.so instead:
the same kernels with their bounds guards compiled in (include/flux.h).
"""

from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import torch

_LIB_PATH = os.path.join(
    os.path.dirname(os.path.abspath(__file__)), "lib",
    "libflux_checked.so" if os.environ.get("FLUX_CHECKED") == "1" else "libflux.so")

FLUX_OK = 0
FLUX_ERR_INVALID_ARG = 1
FLUX_ERR_UNSUPPORTED = 2
FLUX_ERR_CAPACITY = 3
FLUX_ERR_TIMEOUT = 4
FLUX_ERR_CUDA = 5
FLUX_ERR_WORKSPACE = 6

FLUX_DEVICE_CAPACITY = 0x1
FLUX_DEVICE_TIMEOUT = 0x2
FLUX_DEVICE_BAD_LENGTH = 0x4
FLUX_DEVICE_RING_ROUTE = 0x8
FLUX_DEVICE_LAYOUT = 0x10
FLUX_DEVICE_BOUNDS = 0x20

# every entry point declared in include/flux.h
EXPORTED = (
    "flux_mask_words", "flux_route", "flux_kv_append", "flux_prefill",
    "flux_decode_workspace_size", "flux_decode", "flux_sa_block_ranges",
    "flux_get_device_status", "flux_status_string", "flux_version", "flux_decode_static",
    "flux_kv_compact_ring", "flux_kv_append_ring", "flux_decode_ring",
    "flux_selftest_wait_timeout", "flux_prefill_tile_plan", "flux_decode_append",
    "flux_decode_append_ring", "flux_selftest_bounds", "flux_build_checked",
)

# flag bit of a flux_prefill_tile_plan entry: the kernel masks keys of that tile
FLUX_TILE_MASKED = 0x40000000

# bytes of the scratch array flux_decode_static keeps inside the library
FLUX_DECODE_STATIC_SCRATCH_BYTES = 32 * 1024 * 1024


class FluxError(RuntimeError):
    def __init__(self, fn: str, status: int, message: str):
        super().__init__(f"{fn} failed: status {status} ({message})")
        self.status = status


class FluxAttnCfg(ctypes.Structure):
    _fields_ = [("n_layers", ctypes.c_int32), ("n_q_heads", ctypes.c_int32),
                ("n_kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("block", ctypes.c_int32), ("sink", ctypes.c_int32),
                ("window", ctypes.c_int32)]


class FluxRouterWeights(ctypes.Structure):
    _fields_ = [("w1", ctypes.c_void_p), ("b1", ctypes.c_void_p), ("w2", ctypes.c_void_p),
                ("b2", ctypes.c_void_p), ("hidden", ctypes.c_int32),
                ("rank", ctypes.c_int32), ("n_layers", ctypes.c_int32)]


@dataclass(frozen=True)
class AttnCfg:
    """Attention geometry (mirrors flux_attn_cfg)."""
    n_layers: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    block: int
    sink: int
    window: int

    def c(self) -> FluxAttnCfg:
        return FluxAttnCfg(self.n_layers, self.n_q_heads, self.n_kv_heads, self.head_dim,
                           self.block, self.sink, self.window)

    @property
    def mask_words(self) -> int:
        return (self.n_layers + 31) // 32


_lib = None


def library_path() -> str:
    return _LIB_PATH


def lib() -> ctypes.CDLL:
    """Load libflux.so (once).  Raises if it is missing: there is no fallback."""
    global _lib
    if _lib is None:
        if not os.path.exists(_LIB_PATH):
            raise RuntimeError(
                f"libflux.so not found at {_LIB_PATH}; build it with "
                "`python -m sparse_attention_layer_b200.build` (needs nvcc)")
        L = ctypes.CDLL(_LIB_PATH)
        i32, vp, sz = ctypes.c_int32, ctypes.c_void_p, ctypes.c_size_t
        L.flux_mask_words.argtypes = [i32]
        L.flux_mask_words.restype = i32
        L.flux_version.argtypes = []
        L.flux_version.restype = i32
        L.flux_status_string.argtypes = [ctypes.c_int]
        L.flux_status_string.restype = ctypes.c_char_p
        L.flux_get_device_status.argtypes = [vp, ctypes.POINTER(ctypes.c_uint32)]
        L.flux_get_device_status.restype = ctypes.c_int
        L.flux_route.argtypes = [ctypes.POINTER(FluxRouterWeights), vp, i32, i32, i32,
                                 ctypes.c_float, vp, vp, vp]
        L.flux_route.restype = ctypes.c_int
        L.flux_kv_append.argtypes = [ctypes.POINTER(FluxAttnCfg), vp, vp, vp, i32, i32, vp, vp,
                                     i32, vp]
        L.flux_kv_append.restype = ctypes.c_int
        L.flux_prefill.argtypes = [ctypes.POINTER(FluxAttnCfg), i32, vp, vp, vp, vp, vp, i32, i32,
                                   i32, vp, vp]
        L.flux_prefill.restype = ctypes.c_int
        L.flux_decode_workspace_size.argtypes = [ctypes.POINTER(FluxAttnCfg), i32]
        L.flux_decode_workspace_size.restype = sz
        L.flux_decode.argtypes = [ctypes.POINTER(FluxAttnCfg), i32, vp, vp, vp, vp, vp, i32, i32,
                                  vp, vp, sz, vp]
        L.flux_decode.restype = ctypes.c_int
        L.flux_decode_append.argtypes = [ctypes.POINTER(FluxAttnCfg), i32, vp, vp, vp, vp, vp,
                                         vp, vp, i32, i32, vp, vp, sz, vp]
        L.flux_decode_append.restype = ctypes.c_int
        L.flux_decode_append_ring.argtypes = [ctypes.POINTER(FluxAttnCfg), i32, vp, vp, vp, vp,
                                              vp, vp, vp, i32, i32, vp, vp, sz, vp]
        L.flux_decode_append_ring.restype = ctypes.c_int
        L.flux_decode_static.argtypes = [ctypes.POINTER(FluxAttnCfg), i32, vp, vp, vp, vp, vp, i32,
                                         i32, vp, vp]
        L.flux_decode_static.restype = ctypes.c_int
        L.flux_kv_compact_ring.argtypes = [ctypes.POINTER(FluxAttnCfg), vp, vp, i32, vp, i32, vp,
                                           vp, i32, vp]
        L.flux_kv_compact_ring.restype = ctypes.c_int
        L.flux_kv_append_ring.argtypes = [ctypes.POINTER(FluxAttnCfg), vp, vp, vp, i32, i32, vp,
                                          vp, i32, vp]
        L.flux_kv_append_ring.restype = ctypes.c_int
        L.flux_decode_ring.argtypes = [ctypes.POINTER(FluxAttnCfg), i32, vp, vp, vp, vp, vp, i32,
                                       i32, vp, vp, sz, vp]
        L.flux_decode_ring.restype = ctypes.c_int
        L.flux_selftest_wait_timeout.argtypes = [ctypes.c_uint32, vp]
        L.flux_selftest_wait_timeout.restype = ctypes.c_int
        L.flux_selftest_bounds.argtypes = [vp]
        L.flux_selftest_bounds.restype = ctypes.c_int
        L.flux_build_checked.argtypes = []
        L.flux_build_checked.restype = ctypes.c_int
        L.flux_prefill_tile_plan.argtypes = [ctypes.POINTER(FluxAttnCfg), i32, vp, vp, i32, i32,
                                             i32, vp, i32, vp]
        L.flux_prefill_tile_plan.restype = ctypes.c_int
        L.flux_sa_block_ranges.argtypes = [ctypes.POINTER(FluxAttnCfg), i32, vp, vp]
        L.flux_sa_block_ranges.restype = ctypes.c_int
        _lib = L
    return _lib


# ------------------------------------------------------------------ marshalling helpers


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _ptr(t, name: str, dtype, shape=None, allow_none: bool = False):
    if t is None:
        if allow_none:
            return None
        raise ValueError(f"{name} is required")
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor (libflux has no CPU path)")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    return ctypes.c_void_p(t.data_ptr())


def _check(fn: str, status: int) -> None:
    if status != FLUX_OK:
        raise FluxError(fn, status, lib().flux_status_string(status).decode())


# ------------------------------------------------------------------ the ABI, in Python


def flux_mask_words(n_layers: int) -> int:
    return int(lib().flux_mask_words(n_layers))


def flux_version() -> int:
    return int(lib().flux_version())


def flux_status_string(status: int) -> str:
    return lib().flux_status_string(status).decode()


def flux_get_device_status(stream=None) -> int:
    """Read and clear the device status word (FLUX_DEVICE_* bits)."""
    bits = ctypes.c_uint32(0)
    _check("flux_get_device_status", lib().flux_get_device_status(_stream(stream),
                                                                  ctypes.byref(bits)))
    return int(bits.value)


def flux_route(w1, b1, w2, b2, xq, pool_len: int, tau: float, fa_mask, logits=None,
               stream=None) -> None:
    """Layer Router: writes fa_mask [B][mask_words] (int32 storage of the uint32 words)
    and, if given, logits [B][n_layers] float64."""
    rank, hidden = w1.shape
    n_layers = w2.shape[0]
    batch, seq = xq.shape[0], xq.shape[1]
    wts = FluxRouterWeights(
        _ptr(w1, "w1", torch.bfloat16, (rank, hidden)),
        _ptr(b1, "b1", torch.bfloat16, (rank,), allow_none=True),
        _ptr(w2, "w2", torch.bfloat16, (n_layers, rank)),
        _ptr(b2, "b2", torch.bfloat16, (n_layers,), allow_none=True),
        hidden, rank, n_layers)
    st = lib().flux_route(
        ctypes.byref(wts), _ptr(xq, "xq", torch.bfloat16, (batch, seq, hidden)), batch, seq,
        int(pool_len), float(tau),
        _ptr(fa_mask, "fa_mask", torch.int32, (batch, (n_layers + 31) // 32)),
        _ptr(logits, "logits", torch.float64, (batch, n_layers), allow_none=True),
        _stream(stream))
    _check("flux_route", st)


def flux_kv_append(cfg: AttnCfg, k_cache, v_cache, seq_len, k_new, v_new, stream=None) -> None:
    """Append k_new/v_new [B][n][Hkv][d] at seq_len[b] and advance seq_len."""
    batch, hkv, cap, d = k_cache.shape
    n_new = k_new.shape[1]
    c = cfg.c()
    st = lib().flux_kv_append(
        ctypes.byref(c), _ptr(k_cache, "k_cache", torch.bfloat16, (batch, hkv, cap, d)),
        _ptr(v_cache, "v_cache", torch.bfloat16, (batch, hkv, cap, d)),
        _ptr(seq_len, "seq_len", torch.int32, (batch,)), batch, cap,
        _ptr(k_new, "k_new", torch.bfloat16, (batch, n_new, hkv, d)),
        _ptr(v_new, "v_new", torch.bfloat16, (batch, n_new, hkv, d)), n_new, _stream(stream))
    _check("flux_kv_append", st)


def flux_prefill(cfg: AttnCfg, layer: int, fa_mask, q, k_cache, v_cache, seq_len, o,
                 stream=None) -> None:
    """Prefill attention of q [B][n_q][Hq][d] (the last n_q positions) into o."""
    batch, n_q, hq, d = q.shape
    cap = k_cache.shape[2]
    c = cfg.c()
    st = lib().flux_prefill(
        ctypes.byref(c), int(layer), _ptr(fa_mask, "fa_mask", torch.int32, (batch, cfg.mask_words)),
        _ptr(q, "q", torch.bfloat16), _ptr(k_cache, "k_cache", torch.bfloat16,
                                           (batch, cfg.n_kv_heads, cap, d)),
        _ptr(v_cache, "v_cache", torch.bfloat16, (batch, cfg.n_kv_heads, cap, d)),
        _ptr(seq_len, "seq_len", torch.int32, (batch,)), batch, cap, n_q,
        _ptr(o, "o", torch.bfloat16, (batch, n_q, hq, d)), _stream(stream))
    _check("flux_prefill", st)


def flux_decode_workspace_size(cfg: AttnCfg, batch: int) -> int:
    c = cfg.c()
    return int(lib().flux_decode_workspace_size(ctypes.byref(c), int(batch)))


def flux_decode(cfg: AttnCfg, layer: int, fa_mask, q, k_cache, v_cache, seq_len, o, workspace,
                stream=None) -> None:
    """One decode step: q [B][Hq][d] at position seq_len[b]-1 -> o [B][Hq][d]."""
    batch, hq, d = q.shape
    cap = k_cache.shape[2]
    c = cfg.c()
    st = lib().flux_decode(
        ctypes.byref(c), int(layer), _ptr(fa_mask, "fa_mask", torch.int32, (batch, cfg.mask_words)),
        _ptr(q, "q", torch.bfloat16), _ptr(k_cache, "k_cache", torch.bfloat16,
                                           (batch, cfg.n_kv_heads, cap, d)),
        _ptr(v_cache, "v_cache", torch.bfloat16, (batch, cfg.n_kv_heads, cap, d)),
        _ptr(seq_len, "seq_len", torch.int32, (batch,)), batch, cap,
        _ptr(o, "o", torch.bfloat16, (batch, hq, d)),
        _ptr(workspace, "workspace", torch.uint8), workspace.numel(), _stream(stream))
    _check("flux_decode", st)


def flux_decode_append(cfg: AttnCfg, layer: int, fa_mask, q, k_new, v_new, k_cache, v_cache,
                       seq_len, o, workspace, stream=None) -> None:
    """One decode step with its KV append in one launch: k_new/v_new [B][1][Hkv][d] go to
    position seq_len[b], seq_len advances, q [B][Hq][d] attends -> o.  The workspace
    must have been zero-filled once."""
    batch, hq, d = q.shape
    cap = k_cache.shape[2]
    c = cfg.c()
    st = lib().flux_decode_append(
        ctypes.byref(c), int(layer), _ptr(fa_mask, "fa_mask", torch.int32, (batch, cfg.mask_words)),
        _ptr(q, "q", torch.bfloat16),
        _ptr(k_new, "k_new", torch.bfloat16, (batch, 1, cfg.n_kv_heads, d)),
        _ptr(v_new, "v_new", torch.bfloat16, (batch, 1, cfg.n_kv_heads, d)),
        _ptr(k_cache, "k_cache", torch.bfloat16, (batch, cfg.n_kv_heads, cap, d)),
        _ptr(v_cache, "v_cache", torch.bfloat16, (batch, cfg.n_kv_heads, cap, d)),
        _ptr(seq_len, "seq_len", torch.int32, (batch,)), batch, cap,
        _ptr(o, "o", torch.bfloat16, (batch, hq, d)),
        _ptr(workspace, "workspace", torch.uint8), workspace.numel(), _stream(stream))
    _check("flux_decode_append", st)


def flux_decode_append_ring(cfg: AttnCfg, layer: int, fa_mask, q, k_new, v_new, k_ring, v_ring,
                            seq_len, o, workspace, stream=None) -> None:
    """flux_decode_append over an SA layer's ring caches [B][Hkv][sink + ring_rows][d]."""
    batch, hq, d = q.shape
    rows = k_ring.shape[2]
    c = cfg.c()
    st = lib().flux_decode_append_ring(
        ctypes.byref(c), int(layer), _ptr(fa_mask, "fa_mask", torch.int32, (batch, cfg.mask_words)),
        _ptr(q, "q", torch.bfloat16),
        _ptr(k_new, "k_new", torch.bfloat16, (batch, 1, cfg.n_kv_heads, d)),
        _ptr(v_new, "v_new", torch.bfloat16, (batch, 1, cfg.n_kv_heads, d)),
        _ptr(k_ring, "k_ring", torch.bfloat16, (batch, cfg.n_kv_heads, rows, d)),
        _ptr(v_ring, "v_ring", torch.bfloat16, (batch, cfg.n_kv_heads, rows, d)),
        _ptr(seq_len, "seq_len", torch.int32, (batch,)), batch, rows - cfg.sink,
        _ptr(o, "o", torch.bfloat16, (batch, hq, d)),
        _ptr(workspace, "workspace", torch.uint8), workspace.numel(), _stream(stream))
    _check("flux_decode_append_ring", st)


def new_decode_workspace(cfg: AttnCfg, batch: int, device="cuda") -> torch.Tensor:
    """A decode workspace for cfg and batch, zero-filled as the library requires."""
    return torch.zeros(flux_decode_workspace_size(cfg, batch), dtype=torch.uint8, device=device)


def flux_decode_static(cfg: AttnCfg, layer: int, fa_mask, q, k_cache, v_cache, seq_len, o,
                       stream=None) -> None:
    """flux_decode without a workspace argument, for callers that cannot allocate
    device memory: the library's own fixed scratch array (FLUX_DECODE_STATIC_SCRATCH_BYTES)
    holds the split partials.  Calls that overlap on the GPU share that array and race;
    the first call on a device should come before any stream capture."""
    batch, hq, d = q.shape
    cap = k_cache.shape[2]
    c = cfg.c()
    st = lib().flux_decode_static(
        ctypes.byref(c), int(layer), _ptr(fa_mask, "fa_mask", torch.int32, (batch, cfg.mask_words)),
        _ptr(q, "q", torch.bfloat16), _ptr(k_cache, "k_cache", torch.bfloat16,
                                           (batch, cfg.n_kv_heads, cap, d)),
        _ptr(v_cache, "v_cache", torch.bfloat16, (batch, cfg.n_kv_heads, cap, d)),
        _ptr(seq_len, "seq_len", torch.int32, (batch,)), batch, cap,
        _ptr(o, "o", torch.bfloat16, (batch, hq, d)), _stream(stream))
    _check("flux_decode_static", st)


def flux_kv_compact_ring(cfg: AttnCfg, k_cache, v_cache, seq_len, k_ring, v_ring,
                         stream=None) -> None:
    """Copy the rows an SA layer still needs from a full cache [B][Hkv][cap][d] into
    ring caches [B][Hkv][sink + ring_rows][d]."""
    batch, hkv, cap, d = k_cache.shape
    rows = k_ring.shape[2]
    c = cfg.c()
    st = lib().flux_kv_compact_ring(
        ctypes.byref(c), _ptr(k_cache, "k_cache", torch.bfloat16, (batch, hkv, cap, d)),
        _ptr(v_cache, "v_cache", torch.bfloat16, (batch, hkv, cap, d)), cap,
        _ptr(seq_len, "seq_len", torch.int32, (batch,)), batch,
        _ptr(k_ring, "k_ring", torch.bfloat16, (batch, hkv, rows, d)),
        _ptr(v_ring, "v_ring", torch.bfloat16, (batch, hkv, rows, d)), rows - cfg.sink,
        _stream(stream))
    _check("flux_kv_compact_ring", st)


def flux_kv_append_ring(cfg: AttnCfg, k_ring, v_ring, seq_len, k_new, v_new,
                        stream=None) -> None:
    """Append k_new/v_new [B][n][Hkv][d] to ring caches and advance seq_len."""
    batch, hkv, rows, d = k_ring.shape
    n_new = k_new.shape[1]
    c = cfg.c()
    st = lib().flux_kv_append_ring(
        ctypes.byref(c), _ptr(k_ring, "k_ring", torch.bfloat16, (batch, hkv, rows, d)),
        _ptr(v_ring, "v_ring", torch.bfloat16, (batch, hkv, rows, d)),
        _ptr(seq_len, "seq_len", torch.int32, (batch,)), batch, rows - cfg.sink,
        _ptr(k_new, "k_new", torch.bfloat16, (batch, n_new, hkv, d)),
        _ptr(v_new, "v_new", torch.bfloat16, (batch, n_new, hkv, d)), n_new, _stream(stream))
    _check("flux_kv_append_ring", st)


def flux_decode_ring(cfg: AttnCfg, layer: int, fa_mask, q, k_ring, v_ring, seq_len, o,
                     workspace, stream=None) -> None:
    """flux_decode of an SA layer whose cache was compacted into a ring."""
    batch, hq, d = q.shape
    rows = k_ring.shape[2]
    c = cfg.c()
    st = lib().flux_decode_ring(
        ctypes.byref(c), int(layer), _ptr(fa_mask, "fa_mask", torch.int32, (batch, cfg.mask_words)),
        _ptr(q, "q", torch.bfloat16), _ptr(k_ring, "k_ring", torch.bfloat16,
                                           (batch, cfg.n_kv_heads, rows, d)),
        _ptr(v_ring, "v_ring", torch.bfloat16, (batch, cfg.n_kv_heads, rows, d)),
        _ptr(seq_len, "seq_len", torch.int32, (batch,)), batch, rows - cfg.sink,
        _ptr(o, "o", torch.bfloat16, (batch, hq, d)),
        _ptr(workspace, "workspace", torch.uint8), workspace.numel(), _stream(stream))
    _check("flux_decode_ring", st)


def flux_selftest_wait_timeout(limit_us: int, stream=None) -> None:
    """Launch a wait that nothing releases; it must time out into FLUX_DEVICE_TIMEOUT."""
    _check("flux_selftest_wait_timeout",
           lib().flux_selftest_wait_timeout(int(limit_us), _stream(stream)))


def flux_selftest_bounds(stream=None) -> None:
    """Launch a bounds guard that refuses its index: FLUX_DEVICE_BOUNDS in the checked
    build, no status bit in the plain build."""
    _check("flux_selftest_bounds", lib().flux_selftest_bounds(_stream(stream)))


def flux_build_checked() -> bool:
    """True when the loaded library is the checked build."""
    return bool(lib().flux_build_checked())


def flux_sa_block_ranges(cfg: AttnCfg, n_qblocks: int, ranges, stream=None) -> None:
    """SA key-block ranges [n_qblocks][3] (int32) as the kernels compute them."""
    c = cfg.c()
    st = lib().flux_sa_block_ranges(
        ctypes.byref(c), int(n_qblocks), _ptr(ranges, "ranges", torch.int32, (n_qblocks, 3)),
        _stream(stream))
    _check("flux_sa_block_ranges", st)


def flux_prefill_tile_plan(cfg: AttnCfg, layer: int, fa_mask, seq_len, capacity: int, n_q: int,
                           tiles, stream=None) -> None:
    """The KV tiles flux_prefill visits: tiles [B][ceil(n_q/128)][max_tiles] int32 gets
    the 128-key tile index of each visited tile (| FLUX_TILE_MASKED where the kernel
    masks keys), -1 after the last."""
    batch = seq_len.shape[0]
    n_mt = (n_q + 127) // 128
    max_tiles = tiles.shape[2]
    c = cfg.c()
    st = lib().flux_prefill_tile_plan(
        ctypes.byref(c), int(layer), _ptr(fa_mask, "fa_mask", torch.int32, (batch, cfg.mask_words)),
        _ptr(seq_len, "seq_len", torch.int32, (batch,)), batch, int(capacity), int(n_q),
        _ptr(tiles, "tiles", torch.int32, (batch, n_mt, max_tiles)), max_tiles, _stream(stream))
    _check("flux_prefill_tile_plan", st)
