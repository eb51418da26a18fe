"""flux_decode_static: decode for callers that cannot allocate device memory.

Some callers cannot hand the library a workspace -- plugin hosts that give an op no
scratch argument, real-time serving loops that forbid allocation once running, code
that runs while another component owns the device allocator.  flux_decode_static
serves them from a fixed scratch array inside the library.  This test calls it
through the C ABI (ctypes binding) twice in a row and checks each result against
flux_decode with a caller workspace.  Both run the same kernels with the same split
plan and arithmetic, so the outputs must be identical, bit for bit (a stricter demand
than the parity tests' attention tolerance).  It also checks that a call after the
first one reserves no device memory.  It lives in a file of its own, collected last,
and passes alone in a fresh process as well as after the other tests.
"""

import ctypes

import pytest
import torch

from sparse_attention_layer_b200 import flux, inputs
from sparse_attention_layer_b200.flux import AttnCfg
from tests.gpu_cases import CacheCase, mask_words

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _needs_gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    flux.flux_get_device_status()


def test_static_scratch_decode_matches_workspace_decode():
    # Llama-3.1-8B attention geometry, mixed routes, ragged contexts
    cfg = AttnCfg(2, 32, 8, 128, 128, 128, 2048)
    ctx = [5000, 300, 2200, 4097]
    batch = len(ctx)
    case = CacheCase(cfg, ctx, 6000, seed=4242)
    mask = mask_words(batch, cfg.n_layers, [[0], [], [0, 1], []]).cuda()
    ws = flux.new_decode_workspace(cfg, batch)
    qs = [inputs.normal_bf16((batch, cfg.n_q_heads, cfg.head_dim), 9000 + call).cuda()
          for call in range(2)]
    o_ws = [torch.empty_like(q) for q in qs]
    o_static = [torch.full_like(q, float("nan")) for q in qs]
    free = []
    for call, layer in enumerate((0, 1)):   # two calls in a row
        flux.flux_decode(cfg, layer, mask, qs[call], case.k, case.v, case.seq_len, o_ws[call], ws)
        torch.cuda.synchronize()
        free.append(torch.cuda.mem_get_info()[0])
        flux.flux_decode_static(cfg, layer, mask, qs[call], case.k, case.v, case.seq_len,
                                o_static[call])
        torch.cuda.synchronize()
        assert torch.equal(o_static[call], o_ws[call]), f"static-scratch decode, call {call}"
    # the first call may load the library's decode module (and its scratch array); the
    # second one reserves nothing more
    assert torch.cuda.mem_get_info()[0] == free[1]
    assert flux.flux_get_device_status() == 0


def test_static_scratch_rejects_oversized_request():
    # 32 sequences of the Llama geometry need 34 MB of partials: more than the array
    cfg = AttnCfg(2, 32, 8, 128, 128, 128, 2048)
    assert flux.flux_decode_workspace_size(cfg, 32) > flux.FLUX_DECODE_STATIC_SCRATCH_BYTES
    assert flux.flux_decode_workspace_size(cfg, 31) <= flux.FLUX_DECODE_STATIC_SCRATCH_BYTES
    c = cfg.c()
    fake = ctypes.c_void_p(1 << 20)
    st = flux.lib().flux_decode_static(ctypes.byref(c), 0, fake, fake, fake, fake, fake, 32, 4096,
                                       fake, None)
    assert st == flux.FLUX_ERR_WORKSPACE
