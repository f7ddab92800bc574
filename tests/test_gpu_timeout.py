"""The device-side time-out path, exercised without a GPU fault.

The test-only build libflashblock_testhooks.so (the library's own sources,
compiled with FB_TEST_HOOKS) bounds every pipeline wait by 2 ms instead of
1 s, and fb_test_set_skip_k1(1) makes the attention kernels' K producer leave
the load of the second key tile out.  The MMA warp's wait for that tile then
runs out: the CTA records FB_ERR_DEVICE_TIMEOUT in the status word, its other
warps give up their waits, its own copies and MMAs are drained, tensor memory
is freed and the kernel returns.  The next call in the same process must run
normally and match the oracle: the context is still usable."""
import ctypes

import numpy as np
import pytest
import torch

import gpu_cases
from block_diffusion_attention_b200 import flashblock as fbl
from block_diffusion_attention_b200 import synth
from block_diffusion_attention_b200.build import TEST_LIB
from oracle import flashblock_oracle as ora

pytestmark = pytest.mark.gpu

FB_ERR_DEVICE_TIMEOUT = 6


def _testlib():
    lib = ctypes.CDLL(TEST_LIB)
    P, SZ = ctypes.c_void_p, ctypes.c_size_t
    lib.fb_prefix_partial.restype = ctypes.c_int32
    lib.fb_prefix_partial.argtypes = [ctypes.POINTER(fbl.fb_desc), P, P, P, P, P, P, P, SZ, P, P]
    lib.fb_test_set_skip_k1.restype = None
    lib.fb_test_set_skip_k1.argtypes = [ctypes.c_int32]
    return lib


# 32 block tokens x 4 heads = one 128-row query tile (the one-tile kernel);
# 64 tokens = two tiles (the two-tile kernel).  One CTA, eight key tiles.
@pytest.mark.parametrize("block_len", [32, 64])
def test_wait_time_out_is_reported_and_the_next_call_runs(block_len):
    w = synth.WORKLOADS["lm_gqa"].scaled(num_q_heads=4, num_kv_heads=1, block_len=block_len, prefix_len=1024,
                                         blocks=1, steps=1)
    K, V, lens = synth.prefix_kv(w)
    Kt, K64 = gpu_cases.tensors(w, K)
    Vt, V64 = gpu_cases.tensors(w, V)
    layer = gpu_cases.make_layer(w, num_splits=1)
    layer.load_prefix(Kt, Vt, lens)
    Q, _, _ = synth.step_inputs(w, 0, 0)
    Qt, Q64 = gpu_cases.tensors(w, Q)
    lib = _testlib()
    ws = layer.workspace

    def prefix_pass():
        return lib.fb_prefix_partial(ctypes.byref(layer.desc), Qt.data_ptr(), layer.K.data_ptr(), layer.V.data_ptr(),
                                     None, layer.O_pre.data_ptr(), layer.LSE_pre.data_ptr(),
                                     None if ws is None else ws.data_ptr(), 0 if ws is None else ws.numel() * 4,
                                     layer.status.data_ptr(), torch.cuda.current_stream().cuda_stream)

    torch.cuda.synchronize()
    lib.fb_test_set_skip_k1(1)
    try:
        assert prefix_pass() == 0  # the launch itself is fine
        torch.cuda.synchronize()
        assert int(layer.status.item()) == FB_ERR_DEVICE_TIMEOUT
    finally:
        lib.fb_test_set_skip_k1(0)
    layer.status.zero_()
    assert prefix_pass() == 0
    torch.cuda.synchronize()
    assert int(layer.status.item()) == 0
    ref_o, ref_l = ora.prefix_partial(Q64, K64, V64, lens.astype(np.int64), w.softmax_scale)
    gpu_cases.compare("O_pre after a time-out", layer.O_pre.cpu().numpy(), ref_o, w.dtype)
    gpu_cases.compare("LSE_pre after a time-out", layer.LSE_pre.cpu().numpy(), ref_l, w.dtype)
