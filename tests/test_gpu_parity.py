"""GPU parity: the CUDA path against the float64 oracle, element by element, on
scaled-down versions of the five workloads that still span several key and
query tiles with ragged tails, plus the edge cases of the method.  Every call
goes through the C ABI."""
import math

import numpy as np
import pytest
import torch

import gpu_cases
from block_diffusion_attention_b200 import synth
from oracle import flashblock_oracle as ora
from block_diffusion_attention_b200 import flashblock as fbl

pytestmark = pytest.mark.gpu

W = synth.WORKLOADS


def test_tiny_fp32_full_config():
    # the tiny workload is small enough to run at its full size
    gpu_cases.run_workload(W["tiny_fp32"])


def test_tiny_fp32_ragged_multiblock():
    w = W["tiny_fp32"].scaled(prefix_len=301, block_len=13, blocks=2, steps=3, num_q_heads=4, num_kv_heads=2,
                              head_dim=128)
    gpu_cases.run_workload(w)


def test_lm_gqa_scaled_two_blocks():
    w = W["lm_gqa"].scaled(prefix_len=1000, blocks=2, steps=3)
    gpu_cases.run_workload(w)


@pytest.mark.parametrize("num_splits", [1, 3, 7])
def test_lm_gqa_split_counts(num_splits):
    w = W["lm_gqa"].scaled(prefix_len=1500, blocks=1, steps=2)
    gpu_cases.run_workload(w, num_splits=num_splits)


@pytest.mark.parametrize("page_size", [64, 128, 256])
def test_paged_cache(page_size):
    w = W["lm_gqa"].scaled(prefix_len=900, blocks=2, steps=2, num_q_heads=16, num_kv_heads=4)
    gpu_cases.run_workload(w, page_size=page_size)


def test_video_scaled_mha_ragged_rows():
    # G = 1: each 128-row query tile is 128 tokens of one head; 300 = 2*128 + 44
    w = W["video"].scaled(num_q_heads=2, num_kv_heads=2, block_len=300, prefix_len=700, steps=2)
    gpu_cases.run_workload(w)


def test_batched_sparse_scaled():
    w = W["batched_sparse"].scaled(batch=3, num_q_heads=8, num_kv_heads=2, prefix_len=1500,
                                   prefix_min=600, topk=3, steps=5)
    gpu_cases.run_workload(w)


def test_sparse_topk_covers_all_chunks_equals_dense():
    w = W["batched_sparse"].scaled(batch=2, num_q_heads=8, num_kv_heads=2, prefix_len=700,
                                   prefix_min=300, topk=8, steps=1)
    gpu_cases.run_workload(w)


@pytest.mark.parametrize("L,S,G", [(0, 32, 4), (1, 32, 4), (127, 1, 4), (129, 7, 4), (255, 33, 2),
                                   (257, 16, 8), (130, 64, 1)])
def test_edge_lengths(L, S, G):
    w = W["lm_gqa"].scaled(prefix_len=L, block_len=S, num_q_heads=2 * G, num_kv_heads=2, blocks=2, steps=2)
    gpu_cases.run_workload(w)


@pytest.mark.parametrize("B,L,S,G", [(1, 300, 32, 32), (1, 200, 16, 64), (1, 150, 130, 32), (3, 260, 64, 32)])
def test_wide_groups(B, L, S, G):
    # 32 and 64 query heads per kv head: a 128-row query tile holds 4 or 2
    # tokens of one group in the prefix pass; the step runs the 16-row MMA
    # kernel (the first two), the tcgen05 kernel (S > 64, ragged query tiles)
    # and the 128-row MMA kernel (the last)
    w = W["lm_gqa"].scaled(batch=B, prefix_len=L, block_len=S, num_q_heads=2 * G, num_kv_heads=2, blocks=2,
                           steps=2)
    gpu_cases.run_workload(w)


@pytest.mark.parametrize("page_size,num_splits", [(64, 0), (128, 3), (0, 5)])
def test_two_tile_kernel_paged_and_split(page_size, num_splits):
    # units of three query tiles (G = 1, 300 tokens = 2 x 128 + 44): a tile
    # pair plus a lone ragged tile on the two-tile kernel, with paged caches
    # and explicit key splits (prefix pass and uncached pass), two blocks with
    # the append in between
    w = W["video"].scaled(num_q_heads=2, num_kv_heads=2, block_len=300, prefix_len=1500, steps=2, blocks=2)
    gpu_cases.run_workload(w, page_size=page_size, num_splits=num_splits)


@pytest.mark.parametrize("Hq,Hkv,S", [(80, 80, 256), (80, 40, 192)])
def test_two_tile_prefix_pass_tail_split(Hq, Hkv, S):
    # 160 units of two-tile CTAs on a GPU of 148 SMs: a last wave of 12, whose
    # units the prefix pass splits over their keys (into slots the combine
    # merges) while the first 148 write the cached pair directly.  G = 1 with
    # one tile pair per unit, and G = 2 with three tiles (a pair and a lone
    # ragged tile) per unit.
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    w = W["lm_gqa"].scaled(batch=2, num_q_heads=Hq, num_kv_heads=Hkv, block_len=S, prefix_len=1500, steps=2,
                           blocks=1)
    rt = -(-S * (Hq // Hkv) // 128)
    units = w.batch * Hkv * ((rt + 1) // 2)
    tail = units % sms
    if not (units > sms and 0 < 2 * tail <= sms):
        pytest.skip(f"{units} units on {sms} SMs leave no small last wave")
    K, V, lens = synth.prefix_kv(w)
    Kt, K64 = gpu_cases.tensors(w, K)
    Vt, V64 = gpu_cases.tensors(w, V)
    layer = gpu_cases.make_layer(w)
    layer.load_prefix(Kt, Vt, lens)
    k = min(sms // tail, -(-layer.desc.kv_capacity // 128) // 3, 32)
    assert k >= 2
    # A workspace that holds the tail slots only -- (tail unit, split, tile) x
    # 128 rows x (D + 1) floats -- and not the f32 partials of a uniform key
    # split: the call succeeds only on the one-split plan, which takes the
    # tail split when its slots fit.
    tail_bytes = tail * k * 2 * 128 * 129 * 4
    ws = torch.empty(tail_bytes, dtype=torch.uint8, device="cuda")
    Q, _, _ = synth.step_inputs(w, 0, 0)
    Qt, Q64 = gpu_cases.tensors(w, Q)
    fbl.fb_prefix_partial(layer.desc, Qt, layer.K, layer.V, None, layer.O_pre, layer.LSE_pre, ws, layer.status)
    layer.check()
    ref_o, ref_l = ora.prefix_partial(Q64, K64, V64, lens.astype(np.int64), w.softmax_scale, None, 0)
    gpu_cases.compare("O_pre", layer.O_pre.cpu().numpy(), ref_o, w.dtype)
    gpu_cases.compare("LSE_pre", layer.LSE_pre.cpu().numpy(), ref_l, w.dtype)
    del layer, ws
    # the whole cached schedule and the uncached pass at this shape
    gpu_cases.run_workload(w)


def test_two_tile_step_tail_split():
    # a long block (768 tokens, 52 heads, G = 1: three tile pairs per unit,
    # 156 units) on a GPU of 148 SMs: the step's last wave holds 8 units,
    # whose block keys are split 2 ways and merged with the cached pair by
    # the combine (the prefix pass takes its own tail split here too)
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    w = W["video"].scaled(batch=1, num_q_heads=52, num_kv_heads=52, block_len=768, prefix_len=300, steps=2,
                          blocks=1)
    units = 52 * 3
    tail = units % sms
    if not (units > sms and 0 < 2 * tail <= sms and sms // tail >= 2):
        pytest.skip(f"{units} units on {sms} SMs leave no small last wave")
    gpu_cases.run_workload(w)
    # the split path ran: the same step without a workspace (one CTA per
    # unit) agrees to rounding and differs in the tail rows
    K, V, lens = synth.prefix_kv(w)
    Kt, _ = gpu_cases.tensors(w, K)
    Vt, _ = gpu_cases.tensors(w, V)
    layer = gpu_cases.make_layer(w)
    layer.load_prefix(Kt, Vt, lens)
    Q, Kb, Vb = synth.step_inputs(w, 0, 0)
    Qt, _ = gpu_cases.tensors(w, Q)
    Kbt, _ = gpu_cases.tensors(w, Kb)
    Vbt, _ = gpu_cases.tensors(w, Vb)
    layer.refresh(Qt)
    O_split = layer.step(Qt, Kbt, Vbt)
    O_one = torch.empty_like(O_split)
    fbl.fb_block_step(layer.desc, Qt, Kbt, Vbt, layer.O_pre, layer.LSE_pre, O_one, None, layer.status)
    layer.check()
    assert not torch.equal(O_split, O_one)
    assert (O_split.float() - O_one.float()).abs().max().item() < 2e-2


def test_block_step_kernel_choice_both_paths():
    # short blocks with few query rows run the warp-level MMA step kernel with
    # 16 rows per CTA; with more rows than one wave of those CTAs, the one
    # with 128 rows per CTA (16 per warp) -- both against the oracle, the
    # latter also with units whose row count leaves warps without rows (7
    # tokens x 4 heads = 28 rows) and with one-token blocks
    few = W["lm_gqa"].scaled(prefix_len=300, block_len=48, num_q_heads=16, num_kv_heads=2, blocks=1, steps=2)
    many32 = W["lm_gqa"].scaled(batch=12, prefix_len=300, block_len=32, blocks=1, steps=2)
    many48 = W["lm_gqa"].scaled(batch=10, prefix_len=300, block_len=48, num_q_heads=16, num_kv_heads=4,
                                blocks=1, steps=2)
    ragged7 = W["lm_gqa"].scaled(batch=10, prefix_len=300, block_len=7, blocks=2, steps=2)
    one = W["lm_gqa"].scaled(batch=40, prefix_len=129, block_len=1, blocks=2, steps=2)
    for w in (few, many32, many48, ragged7, one):
        gpu_cases.run_workload(w)


def test_edge_lengths_fp32_empty_prefix():
    w = W["tiny_fp32"].scaled(prefix_len=0, block_len=5, steps=2, blocks=2)
    gpu_cases.run_workload(w)


def test_other_softmax_scale():
    # Q ~ N(0,1)/sqrt(D) with the 1/sqrt(D) scale as well: flatter logits
    w = W["lm_gqa"].scaled(prefix_len=800, blocks=1, steps=2, softmax_scale=1.0 / math.sqrt(128))
    gpu_cases.run_workload(w)


def test_large_logits_rescale_path():
    # Q ~ N(0, 4): logits with std ~ 22, so the running row max keeps growing
    # and the lazy rescale of the accumulator fires.  Such a peaked softmax
    # returns single value rows, so the values are scaled by 1/4 (exact in
    # bf16): with |O| up to ~1.2 half an ulp of the bf16 output (2^-9 |O|)
    # stays well below the 2e-2 bound, as it does on the workloads' own
    # distributions (at |O| ~ 4-5 the output's rounding alone would be
    # 1.6e-2).
    w = W["lm_gqa"].scaled(prefix_len=1200, blocks=1, steps=2, q_std=2.0, softmax_scale=1.0)
    gpu_cases.run_workload(w, v_scale=0.25)


def test_refresh_determinism_bitwise():
    w = W["lm_gqa"].scaled(prefix_len=2000, blocks=1, steps=1)
    K, V, lens = synth.prefix_kv(w)
    Kt, _ = gpu_cases.tensors(w, K)
    Vt, _ = gpu_cases.tensors(w, V)
    layer = gpu_cases.make_layer(w)
    layer.load_prefix(Kt, Vt, lens)
    Q, _, _ = synth.step_inputs(w, 0, 0)
    Qt, _ = gpu_cases.tensors(w, Q)
    layer.refresh(Qt)
    a = (layer.O_pre.clone(), layer.LSE_pre.clone())
    layer.refresh(Qt)
    layer.check()
    assert torch.equal(a[0], layer.O_pre) and torch.equal(a[1], layer.LSE_pre)


def test_device_bounds_status_reported():
    # a prefix length past the capacity is reported on the device, not faulted
    w = W["lm_gqa"].scaled(prefix_len=256, blocks=1, steps=1)
    layer = gpu_cases.make_layer(w)
    K, V, lens = synth.prefix_kv(w)
    layer.load_prefix(gpu_cases.tensors(w, K)[0], gpu_cases.tensors(w, V)[0], lens)
    layer.lens.fill_(w.capacity + 5)
    Q, _, _ = synth.step_inputs(w, 0, 0)
    layer.refresh(gpu_cases.tensors(w, Q)[0])
    with pytest.raises(fbl.FlashBlockError) as e:
        layer.check()
    assert e.value.status == 7


def test_block_graph_replay_matches_eager():
    # one block recorded as a CUDA graph replays to the same bits as eager calls
    w = W["lm_gqa"].scaled(prefix_len=1500, blocks=1, steps=3)
    K, V, lens = synth.prefix_kv(w)
    layer = gpu_cases.make_layer(w)
    layer.load_prefix(gpu_cases.tensors(w, K)[0], gpu_cases.tensors(w, V)[0], lens)
    base = synth.block_base(w, 0)
    steps = [tuple(gpu_cases.tensors(w, x)[0] for x in synth.step_inputs(w, 0, s, base)) for s in range(w.steps)]
    eager = [torch.empty_like(steps[0][0]) for _ in range(w.steps)]
    layer.run_block(steps, eager, w.refresh)
    torch.cuda.synchronize()
    outs = [torch.empty_like(steps[0][0]) for _ in range(w.steps)]
    g = layer.capture_block(steps, outs, w.refresh)
    for o in outs:
        o.zero_()
    g.replay()
    layer.check()
    for s in range(w.steps):
        assert torch.equal(outs[s], eager[s]), f"step {s}"


@pytest.mark.parametrize("name,page_size", [("lm_gqa", 0), ("batched_sparse", 0), ("batched_sparse", 128)])
def test_block_graph_advances_the_sequence(name, page_size):
    # one block recorded once and replayed for consecutive blocks: each replay
    # appends the finalized block after the current prefix, advances the
    # device lengths and (sparse prefix) recomputes the touched chunk means,
    # with no host bookkeeping; every step's output, the lengths and the
    # chunk lists follow the oracle's run on its own appended cache
    if name == "lm_gqa":
        w = W["lm_gqa"].scaled(prefix_len=700, blocks=4, steps=3)
    else:
        w = W["batched_sparse"].scaled(batch=3, num_q_heads=8, num_kv_heads=2, prefix_len=1500,
                                       prefix_min=600, topk=3, steps=5, blocks=3)
    K, V, lens = synth.prefix_kv(w)
    Kt, K64 = gpu_cases.tensors(w, K)
    Vt, V64 = gpu_cases.tensors(w, V)
    layer = gpu_cases.make_layer(w, page_size=page_size)
    layer.load_prefix(Kt, Vt, lens)

    def block_inputs(blk):
        base = synth.block_base(w, blk)
        return [tuple(gpu_cases.tensors(w, x) for x in synth.step_inputs(w, blk, s, base))
                for s in range(w.steps)]

    inp = block_inputs(0)
    steps = [tuple(x[0] for x in t) for t in inp]  # the tensors the graph reads
    outs = [torch.empty_like(steps[0][0]) for _ in range(w.steps)]
    # block 0 runs eagerly inside capture_block, before the recording
    g = layer.capture_block(steps, outs, w.refresh, append_kv=(steps[-1][1], steps[-1][2]))
    Kc, Vc, lens_o = K64.copy(), V64.copy(), lens.astype(np.int64).copy()
    S = w.block_len
    for blk in range(w.blocks):
        if blk > 0:
            inp = block_inputs(blk)
            for dst, src in zip(steps, inp):
                for d_t, s_t in zip(dst, src):
                    d_t.copy_(s_t[0])
            for o in outs:
                o.zero_()
            g.replay()
        layer.check()
        got = [o.float().cpu().numpy() for o in outs]
        pre, idx = None, None
        for s in range(w.steps):
            Q64, Kb64, Vb64 = (x[1] for x in inp[s])
            if s in w.refresh or pre is None:
                if w.topk:
                    Km, valid = ora.chunk_means(Kc, lens_o, w.chunk_size)
                    idx = ora.select_chunks(Q64, Km, valid, w.topk)
                pre = ora.prefix_partial(Q64, Kc, Vc, lens_o, w.softmax_scale, idx, w.chunk_size)
            o_ref, _ = ora.block_step(Q64, Kb64, Vb64, pre[0], pre[1], w.softmax_scale)
            gpu_cases.compare(f"graph block {blk} step {s}", got[s], o_ref, w.dtype)
        if w.topk:
            assert np.array_equal(layer.chunk_idx.cpu().numpy(), idx), f"block {blk}: chunk lists"
        # the oracle's own append of the block's last step
        Kb64, Vb64 = inp[-1][1][1], inp[-1][2][1]
        for b in range(w.batch):
            L = int(lens_o[b])
            if L + S <= Kc.shape[1]:
                Kc[b, L:L + S] = Kb64[b]
                Vc[b, L:L + S] = Vb64[b]
                lens_o[b] = L + S
        assert np.array_equal(layer.lens.cpu().numpy(), lens_o), f"block {blk}: prefix lengths"
    if w.topk:
        # the means kept current by the replays equal the means of the grown cache
        Km, _ = ora.chunk_means(Kc, lens_o, w.chunk_size)
        gpu_cases.compare("chunk means after the replays", layer.Kmean.cpu().numpy(), Km, "fp32")


@pytest.mark.parametrize("batch,page_size,block_len,wl", [(1, 0, 32, "lm_gqa"), (1, 64, 32, "lm_gqa"),
                                                          (12, 0, 32, "lm_gqa"), (12, 128, 32, "lm_gqa"),
                                                          (2, 0, 100, "lm_gqa"), (2, 0, 16, "tiny_fp32")])
def test_step_append_equals_step_then_append(batch, page_size, block_len, wl):
    # the block's last step with its append fused into the step kernel (the
    # 16-row kernel at batch 1, the 128-row kernel at batch 12; a 100-token
    # block and the fp32 path run the step and the append one after the
    # other): the same output, cache rows and lengths as fb_block_step then
    # fb_kv_append
    w = W[wl].scaled(batch=batch, prefix_len=600, prefix_min=300, blocks=2, steps=1, block_len=block_len)
    K, V, lens = synth.prefix_kv(w)
    Kt, Vt = gpu_cases.tensors(w, K)[0], gpu_cases.tensors(w, V)[0]
    ref = gpu_cases.make_layer(w, page_size=page_size)
    fused = gpu_cases.make_layer(w, page_size=page_size)
    for layer in (ref, fused):
        layer.load_prefix(Kt, Vt, lens)
    base = synth.block_base(w, 0)
    Q, Kb, Vb = (gpu_cases.tensors(w, x)[0] for x in synth.step_inputs(w, 0, 0, base))
    for layer in (ref, fused):
        layer.refresh(Q)
    o_ref = ref.step(Q, Kb, Vb)
    ref.append(Kb, Vb)
    o_fused = fused.step_append(Q, Kb, Vb)
    ref.check()
    fused.check()
    assert torch.equal(o_fused, o_ref)
    assert torch.equal(fused.lens, ref.lens)
    assert torch.equal(fused.K, ref.K) and torch.equal(fused.V, ref.V)
    # a block that does not fit is reported and not written
    fused.lens.fill_(fbl.fb_cache_rows(fused.desc) - w.block_len + 1)
    before = fused.K.clone()
    fused.step_append(Q, Kb, Vb)
    with pytest.raises(fbl.FlashBlockError) as e:
        fused.check()
    assert e.value.status == 7
    assert torch.equal(fused.K, before)


def test_residual_sparse_reuse():
    # residual reuse: cached unselected-chunk partial + fresh selected chunks + block
    w = W["batched_sparse"].scaled(batch=3, num_q_heads=8, num_kv_heads=2, prefix_len=1500,
                                   prefix_min=600, topk=3, steps=6)
    gpu_cases.run_residual(w)


def test_merge_partials_matches_oracle():
    rng = np.random.default_rng(5)
    B, S, Hq, D = 2, 9, 4, 128
    f32 = lambda x: x.astype(np.float32).astype(np.float64)  # noqa: E731
    Oa, Ob = f32(rng.standard_normal((B, S, Hq, D))), f32(rng.standard_normal((B, S, Hq, D)))
    La, Lb = f32(rng.standard_normal((B, Hq, S)) * 4), f32(rng.standard_normal((B, Hq, S)) * 4)
    La[0, 0, 0] = -np.inf
    La[1, 2, 3] = Lb[1, 2, 3] = -np.inf
    d = fbl.make_desc(B, Hq, Hq, D, S)
    t = lambda x: torch.tensor(x, dtype=torch.float32, device="cuda")  # noqa: E731
    Oo, Lo = torch.empty(B, S, Hq, D, device="cuda"), torch.empty(B, Hq, S, device="cuda")
    fbl.fb_merge_partials(d, t(Oa), t(La), t(Ob), t(Lb), Oo, Lo)
    ref_o, ref_l = ora.merge_partials(Oa, La.transpose(0, 2, 1), Ob, Lb.transpose(0, 2, 1))
    # fp32 on the GPU against float64 from the same (fp32-representable) inputs
    gpu_cases.compare("merge O", Oo.cpu().numpy(), ref_o, "fp32")
    gpu_cases.compare("merge LSE", Lo.cpu().numpy(), ref_l.transpose(0, 2, 1), "fp32")


def _sparse_layer(prefix_len, chunk_size, topk, batch=2):
    w = W["lm_gqa"].scaled(batch=batch, prefix_len=prefix_len, blocks=1, steps=1, chunk_size=chunk_size, topk=topk)
    K, V, lens = synth.prefix_kv(w)
    Kt, K64 = gpu_cases.tensors(w, K)
    Vt, V64 = gpu_cases.tensors(w, V)
    layer = gpu_cases.make_layer(w)
    layer.load_prefix(Kt, Vt, lens)
    Q, _, _ = synth.step_inputs(w, 0, 0)
    Qt, Q64 = gpu_cases.tensors(w, Q)
    return w, layer, Qt, Q64, K64, V64, lens.astype(np.int64)


@pytest.mark.parametrize("dtype,cap,chunk_size,block,G,ties", [
    ("bf16", 3000, 256, 32, 4, False),    # 12 chunk means and 128 query rows: staged in shared memory
    ("fp32", 3000, 256, 32, 4, False),    # the same with fp32 queries
    ("bf16", 2048, 128, 64, 8, False),    # 512 query rows (128 KB) beside the chunk means
    ("bf16", 9000, 128, 32, 4, True),     # 71 chunks, 30 of them with one mean: the tie goes to lower indices
    ("bf16", 33000, 128, 32, 4, True),    # 258 chunks: two lanes per chunk in the rank count
    ("bf16", 70000, 128, 32, 4, False),   # 547 chunk means (274 KB) do not fit: the kernel that streams them
    ("bf16", 70000, 128, 32, 4, True),
])
def test_chunk_selection_kernels(dtype, cap, chunk_size, block, G, ties):
    # fb_select_chunks on given chunk means (no cache needed) against the
    # oracle's top-k of qbar . kbar_c; two lengths per batch leave chunks past
    # the prefix that must not be chosen
    rng = np.random.default_rng(cap + block)
    B, Hkv, D, topk = 2, 2, 128, 16
    Hq = Hkv * G
    nch_total = -(-cap // chunk_size)
    lens = np.array([cap - 5, cap // 2 + 7], np.int32)
    valid = np.arange(nch_total)[None, :] * chunk_size < lens[:, None]
    Km = rng.standard_normal((B, Hkv, nch_total, D)).astype(np.float32)
    if ties:
        # every second of the first 40 chunks carries the same mean, well
        # above the others: equal scores in both float32 and float64, more
        # of them (inside both prefixes) than topk, so the top-k boundary
        # falls inside the tie
        Km *= np.float32(0.01)
        Km[:, :, 0:40:2, :] = rng.standard_normal((B, Hkv, 1, D)).astype(np.float32)
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    Qm = rng.standard_normal((B, block, Hq, D)).astype(np.float32)
    if ties:
        Qm += 2 * Km[:, :, :1, :].repeat(G, axis=1).transpose(0, 2, 1, 3)  # qbar along the tied mean: a high score
    Qt = torch.from_numpy(Qm).to(tdt).cuda()
    lens_t = torch.from_numpy(lens).cuda()
    d = fbl.make_desc(B, Hq, Hkv, D, block, fbl.FB_BF16 if dtype == "bf16" else fbl.FB_FP32, kv_capacity=cap,
                      prefix_lens=lens_t, chunk_size=chunk_size, topk=topk)
    idx = torch.full((B, Hkv, topk), -7, dtype=torch.int32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    fbl.fb_select_chunks(d, Qt, torch.from_numpy(Km).cuda(), idx, status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    Q64 = Qt.float().cpu().numpy().astype(np.float64)
    ref = ora.select_chunks(Q64, Km.astype(np.float64), valid, topk)
    if ties:
        # the tie decides: all of the oracle's picks come from the tied chunks
        sc = ora.chunk_scores(Q64, Km.astype(np.float64), valid)
        for b in range(B):
            for h in range(Hkv):
                assert len(set(sc[b, h, ref[b, h]].tolist())) == 1
    assert np.array_equal(idx.cpu().numpy(), ref)


def test_sparse_chunk_lists_longer_than_a_warp():
    # 40-entry chunk lists (two 32-entry steps of the list scan), hand-made
    # with gaps, against the oracle's prefix partial over the same chunks
    w, layer, Qt, Q64, K64, V64, lens = _sparse_layer(prefix_len=6500, chunk_size=128, topk=40)
    nch = -(-6500 // 128)
    rng = np.random.default_rng(11)
    idx = np.full((w.batch, w.num_kv_heads, w.topk), -1, np.int32)
    for b in range(w.batch):
        for kvh in range(w.num_kv_heads):
            idx[b, kvh] = np.sort(rng.choice(nch, size=w.topk, replace=False))
    idx[1, 3, 35:] = -1  # a shorter list
    layer.chunk_idx.copy_(torch.from_numpy(idx))
    fbl.fb_prefix_partial(layer.desc, Qt, layer.K, layer.V, layer.chunk_idx, layer.O_pre, layer.LSE_pre,
                          layer.workspace, layer.status)
    layer.check()
    ref_o, ref_l = ora.prefix_partial(Q64, K64, V64, lens, w.softmax_scale, idx, w.chunk_size)
    gpu_cases.compare("O_pre", layer.O_pre.cpu().numpy(), ref_o, w.dtype)
    gpu_cases.compare("LSE_pre", layer.LSE_pre.cpu().numpy(), ref_l, w.dtype)


@pytest.mark.parametrize("bad", ["descending", "past_prefix"])
def test_sparse_invalid_chunk_list_reported(bad):
    # a list entry that is not above its predecessor, or lies past the valid
    # prefix, ends the list and is reported; the entries before it are used
    w, layer, Qt, Q64, K64, V64, lens = _sparse_layer(prefix_len=3000, chunk_size=256, topk=6, batch=1)
    idx = np.full((w.batch, w.num_kv_heads, w.topk), -1, np.int32)
    idx[0, :, :3] = [1, 4, 7]
    idx[0, 2, 3] = 2 if bad == "descending" else 40
    idx[0, 2, 4] = 9
    layer.chunk_idx.copy_(torch.from_numpy(idx))
    fbl.fb_prefix_partial(layer.desc, Qt, layer.K, layer.V, layer.chunk_idx, layer.O_pre, layer.LSE_pre,
                          layer.workspace, layer.status)
    with pytest.raises(fbl.FlashBlockError) as e:
        layer.check()
    assert e.value.status == 7
    used = idx.copy()
    used[0, 2, 3:] = -1
    ref_o, ref_l = ora.prefix_partial(Q64, K64, V64, lens, w.softmax_scale, used, w.chunk_size)
    gpu_cases.compare("O_pre", layer.O_pre.cpu().numpy(), ref_o, w.dtype)
    gpu_cases.compare("LSE_pre", layer.LSE_pre.cpu().numpy(), ref_l, w.dtype)
