"""The C-ABI library loads, exports every function its header declares, and
rejects bad arguments on the host before launching anything (CPU only: no
compute call reaches a device here)."""
import ctypes

import pytest

from block_diffusion_attention_b200 import flashblock as fbl


@pytest.fixture(scope="module")
def lib():
    return fbl.load()


def test_exports_every_declared_symbol(lib):
    names = fbl.header_functions()
    assert len(names) >= 11
    for n in names:
        assert hasattr(lib, n), f"{n} declared in flashblock.h but not exported"


def test_test_hooks_only_in_the_test_library(lib):
    # the hook that leaves a K load out lives only in the test-only build
    import os
    from block_diffusion_attention_b200.build import TEST_LIB
    assert not hasattr(lib, "fb_test_set_skip_k1")
    assert os.path.exists(TEST_LIB)
    tl = ctypes.CDLL(TEST_LIB)
    assert hasattr(tl, "fb_test_set_skip_k1")
    for n in fbl.header_functions():
        assert hasattr(tl, n), n


def test_version_and_status_strings(lib):
    assert fbl.fb_abi_version() == fbl.ABI_VERSION == 2
    for code, name in fbl.STATUS.items():
        assert fbl.fb_status_string(code) == name
    assert fbl.fb_status_string(99) == "FB_ERR_UNKNOWN"
    assert fbl.fb_launch_count() >= 0


def _desc(**kw):
    base = dict(batch=1, num_q_heads=32, num_kv_heads=8, head_dim=128, block_len=32,
                dtype=fbl.FB_BF16, softmax_scale=1.0, kv_capacity=8192)
    base.update(kw)
    d = fbl.make_desc(**base)
    d.prefix_lens = 0x10000  # a host-side stand-in; validation never dereferences it
    return d


FAKE = 0x7f0000000000  # 16-byte aligned, never dereferenced


def _prefix(lib, d, q=FAKE, k=FAKE, v=FAKE, idx=None, o=FAKE, l=FAKE, ws=None, wsb=0):
    return lib.fb_prefix_partial(ctypes.byref(d), q, k, v, idx, o, l, ws, wsb, None, None) \
        if d is not None else lib.fb_prefix_partial(None, q, k, v, idx, o, l, ws, wsb, None, None)


def test_host_validation_codes(lib):
    assert _prefix(lib, None) == 1
    assert _prefix(lib, _desc(batch=0)) == 1
    assert _prefix(lib, _desc(num_q_heads=30)) == 1           # not a multiple of Hkv
    assert _prefix(lib, _desc(softmax_scale=0.0)) == 1
    assert _prefix(lib, _desc(softmax_scale=float("nan"))) == 1
    assert _prefix(lib, _desc(head_dim=64)) == 2              # bf16 path is D = 128
    assert _prefix(lib, _desc(num_q_heads=24, num_kv_heads=8)) == 2  # G = 3
    assert _prefix(lib, _desc(dtype=7)) == 2
    assert _prefix(lib, _desc(dtype=fbl.FB_FP32, head_dim=48)) == 2
    assert _prefix(lib, _desc(), q=None) == 1
    assert _prefix(lib, _desc(), q=FAKE + 8) == 3              # TMA needs 16-byte alignment
    assert _prefix(lib, _desc(page_size=100, max_pages=4, num_pages=4, block_table=None)) == 2
    d = _desc(page_size=128, max_pages=4, num_pages=4)
    assert _prefix(lib, d) == 1                                # paged without a block table
    assert _prefix(lib, _desc(topk=4, chunk_size=256)) == 1    # sparse without a chunk list
    assert _prefix(lib, _desc(topk=4, chunk_size=200), idx=FAKE) == 2
    # long prefix -> split-key workspace required
    d = _desc(kv_capacity=131072)
    assert fbl.fb_workspace_bytes(d) > 0
    assert _prefix(lib, d) == 4
    blk = lib.fb_block_step(ctypes.byref(_desc()), FAKE, FAKE, FAKE, FAKE, FAKE, None, None, None, 0, None, None)
    assert blk == 1
    assert lib.fb_chunk_means(ctypes.byref(_desc(chunk_size=256)), FAKE, 0, 999, FAKE, None, None) == 1
    assert lib.fb_select_chunks(ctypes.byref(_desc(chunk_size=256, topk=0)), FAKE, FAKE, FAKE, None, None) == 1
    tail = lib.fb_chunk_means_tail
    assert tail(ctypes.byref(_desc(chunk_size=256)), FAKE, 0, FAKE, None, None) == 1     # rows > 0
    assert tail(ctypes.byref(_desc(chunk_size=0)), FAKE, 32, FAKE, None, None) == 1
    assert tail(ctypes.byref(_desc(chunk_size=256)), FAKE, 32, FAKE + 4, None, None) == 3
    assert lib.fb_kv_append(ctypes.byref(_desc(kv_capacity=0)), FAKE, FAKE, FAKE, FAKE, None, None, None) == 1


def test_workspace_bytes_formula(lib):
    d = _desc(kv_capacity=131072, num_splits=5)
    # splits x rows x (D + 1) floats
    assert fbl.fb_workspace_bytes(d) == 5 * 32 * 32 * 129 * 4
    # fp32 has no split partials: only the threshold policy's per-4-token counts
    assert fbl.fb_workspace_bytes(_desc(dtype=fbl.FB_FP32, head_dim=64)) == 1 * 8 * 4
    assert fbl.fb_workspace_bytes(_desc(dtype=fbl.FB_FP32, head_dim=64, batch=3, block_len=33)) == 3 * 9 * 4
    assert fbl.fb_cache_rows(_desc(page_size=256, max_pages=3, num_pages=9)) == 768


def test_policy_validation_codes(lib):
    d = _desc()
    hw = lib.fb_headwise_refresh_mask
    assert hw(ctypes.byref(d), None, FAKE, ctypes.c_float(0.9), FAKE, None, None) == 1
    assert hw(ctypes.byref(d), FAKE, FAKE, ctypes.c_float(float("nan")), FAKE, None, None) == 1
    assert hw(ctypes.byref(d), FAKE + 8, FAKE, ctypes.c_float(0.9), FAKE, None, None) == 3
    assert hw(ctypes.byref(d), FAKE, FAKE, ctypes.c_float(0.9), FAKE + 2, None, None) == 3
    th = lib.fb_threshold_refresh_mask
    args = (FAKE, FAKE, FAKE, FAKE)
    assert th(ctypes.byref(d), *args, ctypes.c_float(float("nan")), 1, FAKE, None, FAKE, 4096, None) == 1
    assert th(ctypes.byref(d), *args, ctypes.c_float(0.25), 1, None, None, FAKE, 4096, None) == 1
    assert th(ctypes.byref(d), FAKE + 4, FAKE, FAKE, FAKE, ctypes.c_float(0.25), 1, FAKE, None, FAKE, 4096,
              None) == 3
    assert th(ctypes.byref(d), *args, ctypes.c_float(0.25), 1, FAKE, None, None, 0, None) == 4
    assert th(ctypes.byref(d), *args, ctypes.c_float(0.25), 1, FAKE, None, FAKE, 4, None) == 4  # needs 8 * 4
    pm = lib.fb_prefix_partial_masked
    assert pm(ctypes.byref(d), FAKE, FAKE, FAKE, None, None, FAKE, FAKE, None, 0, None, None) == 1
    assert pm(ctypes.byref(d), FAKE, FAKE, FAKE, None, FAKE + 2, FAKE, FAKE, None, 0, None, None) == 3
    assert pm(ctypes.byref(_desc(batch=0)), FAKE, FAKE, FAKE, None, FAKE, FAKE, FAKE, None, 0, None, None) == 1
