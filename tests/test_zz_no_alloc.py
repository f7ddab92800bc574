"""fb_prefix_partial_noalloc: the prefix pass for callers that may not
allocate device memory (an embedding that owns one fixed device arena, a
plug-in host that gives its plug-ins no allocator, a serving loop that cannot
afford the device-wide synchronisation of cudaMalloc/cudaFree).  Its split
partials live in a static array of the library instead of a caller
workspace; its results must match the regular entry point's, call after
call.

Collected last on purpose (test_zz_*): if it fails, a run that stops at the
first failure has already run every other test.  It builds its own inputs, so
it passes alone in a fresh process as well as after the other tests."""
import ctypes

import pytest
import torch

import gpu_cases
from block_diffusion_attention_b200 import flashblock as fbl
from block_diffusion_attention_b200 import synth

pytestmark = pytest.mark.gpu


def test_noalloc_matches_workspace_entry_point_two_calls_in_a_row():
    # 4096-token prefix, 8 kv heads: the prefix pass splits its keys, so the
    # scratch array is really used
    w = synth.WORKLOADS["lm_gqa"].scaled(prefix_len=4096, blocks=1, steps=2)
    layer = gpu_cases.make_layer(w)
    K, V, lens = synth.prefix_kv(w)
    layer.load_prefix(gpu_cases.tensors(w, K)[0], gpu_cases.tensors(w, V)[0], lens)
    assert fbl.fb_workspace_bytes(layer.desc) > 0
    O2 = torch.empty_like(layer.O_pre)
    L2 = torch.empty_like(layer.LSE_pre)
    base = synth.block_base(w, 0)
    for step in range(2):
        Q = gpu_cases.tensors(w, synth.step_inputs(w, 0, step, base)[0])[0]
        layer.refresh(Q)  # regular entry point, caller workspace
        O2.fill_(float("nan"))
        L2.fill_(float("nan"))
        fbl.fb_prefix_partial_noalloc(layer.desc, Q, layer.K, layer.V, None, O2, L2, layer.status)
        layer.check()
        gpu_cases.compare(f"noalloc O_pre, call {step}", O2.cpu().numpy(), layer.O_pre.cpu().numpy(), "bf16")
        gpu_cases.compare(f"noalloc LSE_pre, call {step}", L2.cpu().numpy(), layer.LSE_pre.cpu().numpy(), "bf16")
        # the same kernels with the same split plan and merge order: the
        # results are bit-identical, not just within tolerance
        assert torch.equal(O2, layer.O_pre) and torch.equal(L2, layer.LSE_pre), f"call {step}: not bit-identical"


def test_noalloc_rejects_partials_larger_than_the_scratch():
    # B16 x S64 x Hq32 rows with 4 key splits need ~68 MB of partials
    d = fbl.make_desc(16, 32, 8, 128, 64, kv_capacity=32832)
    lens = torch.zeros(16, dtype=torch.int32, device="cuda")
    d.prefix_lens = lens.data_ptr()
    if fbl.fb_workspace_bytes(d) <= 16 << 20:
        pytest.skip("this GPU's split choice fits the scratch")
    fake = 0x7f0000000000  # never dereferenced: the size check comes first
    st = fbl.load().fb_prefix_partial_noalloc(ctypes.byref(d), fake, fake, fake, None, fake, fake, None, None)
    assert st == 4  # FB_ERR_WORKSPACE
