"""bench.py's JSON line, built on the CPU from a synthetic record of timings:
every key of the benchmark contract is present and the derived figures follow
from the record (no GPU: the timed phases are not run)."""
import argparse
import json
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from block_diffusion_attention_b200 import synth  # noqa: E402


def _args(**kw):
    base = dict(gpus=1, steps=4, warmup=3, workload="long_ctx", impl="ours", no_cpu_baseline=True,
                residual=False, no_graph=False, policy=None, gamma=0.9, tau=None, eps=0.25,
                phases="cached,uncached,e2e")
    base.update(kw)
    return argparse.Namespace(**base)


def _res(w, with_e2e=True, **kw):
    res = {"pre_ms": [0.1, 0.1], "sel_ms": [0.02, 0.02], "blk_ms": [0.005], "lens0": [w.prefix_len] * w.batch,
           "lens1": [w.prefix_len] * w.batch, "ms_cached": 0.6, "ms_cached_eager": 0.7, "ms_unc": 3.0,
           "graph": True, "launches": 44, "clocks": {"sm_mhz": 1965, "sm_max_mhz": 1965, "reasons": []}}
    if with_e2e:
        res.update({"ms_e2e": 1.2, "h2d": 1000, "d2h": 500, "h2d_ms": 0.1, "d2h_ms": 0.05})
    res.update(kw)
    return res


@pytest.mark.parametrize("kw", [{}, {"policy": "headwise"}, {"policy": "threshold", "tau": 5},
                                {"workload": "batched_sparse"}, {"workload": "batched_sparse", "residual": True}])
def test_report_line_has_contract_keys(capsys, kw):
    args = _args(**kw)
    w = synth.WORKLOADS[args.workload].scaled(blocks=1)
    bench.report(args, synth.WORKLOADS[args.workload], w, 1, _res(w, refresh_fraction=0.25))
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "roofline", "e2e", "gpu_launches", "clocks"):
        assert key in line, key
    assert line["n_gpus"] == 1 and line["steps"] == 4 and line["higher_is_better"] is True
    # value = B * S tokens per block over the timed blocks
    assert line["value"] == pytest.approx(w.batch * w.block_len * 4 / 0.6e-3)
    roof = line["roofline"]
    assert roof["bound"] in ("hbm", "tensor") and roof["frac"] == pytest.approx(roof["achieved"] / roof["peak"])
    assert line["e2e"]["h2d_bytes_per_step"] == 1000 and line["e2e"]["d2h_bytes_per_step"] == 500
    assert line["e2e"]["h2d_gbs"] == pytest.approx(1000 / 0.1e-3 / 1e9)
    if args.policy:
        assert line["config"]["policy"]["name"] == args.policy
        assert line["refresh_fraction"] == 0.25
    if args.workload == "batched_sparse":
        assert line["chunk_select_us"] == pytest.approx(20.0)
    if args.workload == "long_ctx" and not args.residual:
        # the recorded capture of the current kernel, or null when there is none
        assert roof["traffic"] == bench.recorded_traffic("long_ctx")


def test_recorded_traffic_needs_the_captured_sources(monkeypatch):
    # a capture is reported only while the kernel sources hash to the value
    # recorded with it
    monkeypatch.setattr(bench, "NCU_TRAFFIC", {"long_ctx": {"bytes": 123, "sources": bench.kernel_source_hash()}})
    assert bench.recorded_traffic("long_ctx") == 123
    monkeypatch.setattr(bench, "NCU_TRAFFIC", {"long_ctx": {"bytes": 123, "sources": "0" * 16}})
    assert bench.recorded_traffic("long_ctx") is None
    assert bench.recorded_traffic("video") is None


def test_report_l2_cold_prefix_figure(capsys):
    # a workload whose KV cache fits in L2 reports the prefix pass after an
    # L2 eviction (a scratch read; and a scratch write, dirty lines) beside
    # the warm figure
    args = _args(workload="lm_gqa")
    w = synth.WORKLOADS["lm_gqa"].scaled(blocks=1)
    assert bench.kv_cache_bytes(w) < bench.L2_BYTES
    bench.report(args, synth.WORKLOADS["lm_gqa"], w, 1,
                 _res(w, pre_cold_ms=[0.02, 0.02], pre_cold_dirty_ms=[0.024, 0.026]))
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["prefix_pass_l2_cold_us"] == pytest.approx(20.0)
    assert line["prefix_gbs_l2_cold"] == pytest.approx(bench.prefix_bytes(w, [w.prefix_len]) / 20e-6 / 1e9)
    assert line["prefix_pass_l2_cold_dirty_us"] == pytest.approx(25.0)
    assert "L2" in line["config"]["l2"]


@pytest.mark.parametrize("h2d_ms,d2h_ms,bound", [(0.1, 0.05, "compute"), (0.5, 0.05, "host-to-device copies"),
                                                 (0.1, 0.3, "device-to-host copies")])
def test_report_names_what_bounds_e2e(capsys, h2d_ms, d2h_ms, bound):
    # a block's compute is 0.6 ms / 4 timed blocks = 0.15 ms
    args = _args()
    w = synth.WORKLOADS["long_ctx"].scaled(blocks=1)
    bench.report(args, synth.WORKLOADS["long_ctx"], w, 1, _res(w, h2d_ms=h2d_ms, d2h_ms=d2h_ms))
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["e2e"]["bound_by"] == bound


def test_report_without_e2e_phase(capsys):
    args = _args(phases="cached")
    w = synth.WORKLOADS["long_ctx"].scaled(blocks=1)
    bench.report(args, synth.WORKLOADS["long_ctx"], w, 1, _res(w, with_e2e=False, ms_unc=None))
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["e2e"] is None and line["uncached_us_per_denoise_step"] is None


def test_reference_arm_line(capsys, monkeypatch):
    # the reference arm times the oracle on the host: a real run on the tiny
    # workload (seconds), its line carrying the contract's keys
    monkeypatch.delenv("RANK", raising=False)
    args = _args(workload="tiny_fp32", impl="reference", steps=1, warmup=0)
    assert bench.run_reference(args) == 0
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["unit"] == "tokens/s" and line["value"] > 0
    assert line["higher_is_better"] is True and line["steps"] == 1 and line["warmup"] == 0
    assert line["config"]["workload"].startswith("tiny_fp32")
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == line["value"]
    # the step time is the measured sample's, not scaled up to the whole block
    assert line["ms_per_step"] == pytest.approx(cb["sample_seconds_measured"] * 1e3)
    assert line["value"] == pytest.approx(16 * cb["sample_fraction_of_block"] / cb["sample_seconds_measured"])
    assert line["e2e"] == {"value": line["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}


def test_reference_arm_other_ranks_do_no_work(capsys, monkeypatch):
    monkeypatch.setenv("RANK", "1")
    args = _args(workload="tiny_fp32", impl="reference", steps=1, warmup=0)
    assert bench.run_reference(args) == 0
    assert capsys.readouterr().out.strip() == ""
