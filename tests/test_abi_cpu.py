"""C-ABI library checks that need no GPU: the library builds and loads, exports every
entry point include/flux.h declares, and rejects bad arguments on the host before any
CUDA call.  No compute call is made here."""

import ctypes
import os
import re

import pytest
import torch

from sparse_attention_layer_b200 import build, flux

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    build.build()
    return flux.lib()


def header_functions():
    with open(os.path.join(ROOT, "include", "flux.h")) as f:
        text = f.read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(flux_[a-z_0-9]+)\s*\(", text)))


def test_header_and_binding_agree():
    assert header_functions() == sorted(flux.EXPORTED)


def test_status_constants_agree():
    """Every device status bit and status code the header defines has the same value in
    the binding (the tests and bench.py read them from there)."""
    with open(os.path.join(ROOT, "include", "flux.h")) as f:
        text = f.read()
    bits = dict(re.findall(r"#define (FLUX_DEVICE_[A-Z_]+) (0x[0-9a-fA-F]+)u", text))
    codes = dict(re.findall(r"\b(FLUX_(?:OK|ERR_[A-Z_]+)) = (\d+)", text))
    assert len(bits) >= 5 and len(codes) >= 7
    for name, val in bits.items():
        assert getattr(flux, name) == int(val, 16), name
    for name, val in codes.items():
        assert getattr(flux, name) == int(val), name
    assert len(set(int(v, 16) for v in bits.values())) == len(bits)  # distinct bits


def test_library_exports_every_header_symbol(L):
    for name in header_functions():
        assert hasattr(L, name), f"libflux.so does not export {name}"


def test_checked_build_exports_the_same_entry_points(L):
    """libflux_checked.so (bounds guards compiled in) builds here too, exports every
    header symbol, and says which build it is; the plain library says it is not."""
    path = build.build(checked=True)
    assert path.endswith("libflux_checked.so")
    C = ctypes.CDLL(path)
    for name in header_functions():
        assert hasattr(C, name), f"libflux_checked.so does not export {name}"
    C.flux_build_checked.restype = ctypes.c_int
    L.flux_build_checked.restype = ctypes.c_int
    assert C.flux_build_checked() == 1
    assert L.flux_build_checked() == 0


def test_library_is_sm100a_only(L):
    # the build passes exactly one -gencode, for sm_100a
    assert build.ARCH_FLAGS == ["-gencode", "arch=compute_100a,code=sm_100a"]


def test_host_helpers(L):
    assert flux.flux_mask_words(1) == 1
    assert flux.flux_mask_words(32) == 1
    assert flux.flux_mask_words(33) == 2
    assert flux.flux_mask_words(0) == 0
    assert flux.flux_version() >= 100
    assert flux.flux_status_string(0) == "ok"
    assert "capacity" in flux.flux_status_string(3)
    assert flux.flux_status_string(99) == "unknown status"


def _cfg(**kw):
    base = dict(n_layers=32, n_q_heads=32, n_kv_heads=8, head_dim=128, block=128, sink=128,
                window=2048)
    base.update(kw)
    return flux.AttnCfg(**base).c()


def test_workspace_size_formula(L):
    # 1025 arrival counters padded to 4352 bytes, then per (sequence, KV head, split, query
    # head of the group): d fp32 partials + (max, sum)
    c = _cfg()
    got = L.flux_decode_workspace_size(ctypes.byref(c), 16)
    recs = 16 * 8 * 64 * 4
    assert got == 4352 + (recs * 128 * 4 + 255) // 256 * 256 + recs * 8
    bad = _cfg(head_dim=96)
    assert L.flux_decode_workspace_size(ctypes.byref(bad), 16) == 0
    assert L.flux_decode_workspace_size(ctypes.byref(c), 0) == 0


@pytest.mark.parametrize("kw,status", [
    (dict(n_kv_heads=7), flux.FLUX_ERR_INVALID_ARG),      # Hq % Hkv != 0
    (dict(n_q_heads=48, n_kv_heads=3), flux.FLUX_ERR_UNSUPPORTED),  # group 16
    (dict(head_dim=96), flux.FLUX_ERR_UNSUPPORTED),
    (dict(block=32, sink=64, window=256), flux.FLUX_ERR_UNSUPPORTED),
    (dict(sink=100), flux.FLUX_ERR_INVALID_ARG),          # sink not a block multiple
    (dict(window=0), flux.FLUX_ERR_INVALID_ARG),
    (dict(n_layers=0), flux.FLUX_ERR_INVALID_ARG),
])
def test_prefill_rejects_bad_geometry(L, kw, status):
    c = _cfg(**kw)
    fake = ctypes.c_void_p(1 << 20)
    st = L.flux_prefill(ctypes.byref(c), 0, fake, fake, fake, fake, fake, 1, 1024, 128, fake,
                        None)
    assert st == status


def test_null_and_range_checks(L):
    c = _cfg()
    fake = ctypes.c_void_p(1 << 20)
    assert L.flux_prefill(ctypes.byref(c), 0, None, fake, fake, fake, fake, 1, 1024, 128, fake,
                          None) == flux.FLUX_ERR_INVALID_ARG
    assert L.flux_prefill(ctypes.byref(c), 32, fake, fake, fake, fake, fake, 1, 1024, 128, fake,
                          None) == flux.FLUX_ERR_INVALID_ARG          # layer out of range
    assert L.flux_prefill(ctypes.byref(c), 0, fake, fake, fake, fake, fake, 1, 1024, 2048, fake,
                          None) == flux.FLUX_ERR_INVALID_ARG          # n_q > capacity
    assert L.flux_prefill(ctypes.byref(c), 0, fake, ctypes.c_void_p((1 << 20) + 2), fake, fake,
                          fake, 1, 1024, 128, fake, None) == flux.FLUX_ERR_INVALID_ARG  # unaligned
    assert L.flux_kv_append(ctypes.byref(c), fake, fake, fake, 1, 100, fake, fake, 101,
                            None) == flux.FLUX_ERR_CAPACITY
    assert L.flux_decode(ctypes.byref(c), 0, fake, fake, fake, fake, fake, 1, 1024, fake, None, 0,
                         None) == flux.FLUX_ERR_WORKSPACE
    assert L.flux_decode(ctypes.byref(c), 0, fake, fake, fake, fake, fake, 1, 1024, fake, fake, 16,
                         None) == flux.FLUX_ERR_WORKSPACE
    w = flux.FluxRouterWeights(fake, None, fake, None, 4096, 256, 32)
    assert L.flux_route(ctypes.byref(w), fake, 1, 8192, 100, ctypes.c_float(float("nan")), fake,
                        None, None) == flux.FLUX_ERR_INVALID_ARG
    w.hidden = 4100  # not a multiple of 8
    assert L.flux_route(ctypes.byref(w), fake, 1, 8192, 100, 0.0, fake, None,
                        None) == flux.FLUX_ERR_INVALID_ARG


def test_binding_refuses_cpu_tensors(L):
    cfg = flux.AttnCfg(2, 8, 2, 64, 64, 64, 256)
    k = torch.zeros(1, 2, 128, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="CUDA tensor"):
        flux.flux_kv_append(cfg, k, k, torch.zeros(1, dtype=torch.int32),
                            torch.zeros(1, 4, 2, 64, dtype=torch.bfloat16),
                            torch.zeros(1, 4, 2, 64, dtype=torch.bfloat16))


def test_product_package_never_imports_the_oracle():
    pat = re.compile(r"^\s*(from\s+oracle\b|import\s+oracle\b|from\s+\.\.?oracle)", re.M)
    pkg = os.path.join(ROOT, "sparse_attention_layer_b200")
    for dirpath, _, files in os.walk(pkg):
        for fn in files:
            if fn.endswith(".py"):
                with open(os.path.join(dirpath, fn)) as f:
                    assert not pat.search(f.read()), f"{fn} imports the oracle"


def test_tile_plan_flag_and_host_checks(L):
    with open(os.path.join(ROOT, "include", "flux.h")) as f:
        text = f.read()
    assert int(re.search(r"#define FLUX_TILE_MASKED (0x[0-9a-fA-F]+)", text).group(1), 16) == \
        flux.FLUX_TILE_MASKED
    c = _cfg()
    fake = ctypes.c_void_p(1 << 20)
    # max_tiles must cover ceil(capacity / 128) key tiles
    assert L.flux_prefill_tile_plan(ctypes.byref(c), 0, fake, fake, 1, 1024, 512, fake, 7,
                                    None) == flux.FLUX_ERR_INVALID_ARG
    assert L.flux_prefill_tile_plan(ctypes.byref(c), 0, fake, fake, 1, 1024, 2048, fake, 8,
                                    None) == flux.FLUX_ERR_INVALID_ARG   # n_q > capacity
    assert L.flux_prefill_tile_plan(ctypes.byref(c), 40, fake, fake, 1, 1024, 512, fake, 8,
                                    None) == flux.FLUX_ERR_INVALID_ARG   # layer out of range
    assert L.flux_prefill_tile_plan(ctypes.byref(c), 0, fake, fake, 1, 1024, 0, fake, 8,
                                    None) == flux.FLUX_OK                # nothing to plan


def test_fused_decode_host_checks(L):
    c = _cfg()
    fake = ctypes.c_void_p(1 << 20)
    # missing k_new
    assert L.flux_decode_append(ctypes.byref(c), 0, fake, fake, None, fake, fake, fake, fake, 1,
                                1024, fake, fake, 1 << 30, None) == flux.FLUX_ERR_INVALID_ARG
    # workspace too small
    assert L.flux_decode_append(ctypes.byref(c), 0, fake, fake, fake, fake, fake, fake, fake, 1,
                                1024, fake, fake, 16, None) == flux.FLUX_ERR_WORKSPACE
    # ring shorter than the window
    assert L.flux_decode_append_ring(ctypes.byref(c), 0, fake, fake, fake, fake, fake, fake, fake,
                                     1, 1024, fake, fake, 1 << 30, None) == flux.FLUX_ERR_INVALID_ARG
