"""Host-side arithmetic of bench.py (no GPU): workload tables, call order, the
roofline and throughput formulas, and the fraction-sweep summary, on fake
timings whose answers are known in closed form."""
import argparse
import os
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
import synth_inputs as si  # noqa: E402

PK = {"hbm_gbs": 6000.0, "bf16_tflops": 1500.0, "bf16_tflops_sustained": 1200.0, "source": "test"}


def _args(steps=4):
    return argparse.Namespace(steps=steps, warmup=3)


def _fake_t(ms_total, seg_ms=None, launches=1):
    return {"ms": ms_total, "e2e_ms": 2 * ms_total, "seg_ms": seg_ms, "clocks": {}, "h2d": 10, "d2h": 20,
            "launches": launches}


def test_stack_layers_order_and_fractions():
    layers = bench.build_layers("stack", only=["q", "down"])
    assert len(layers) == 2 * bench.STACK_LAYERS
    calls = bench.calls_of(layers)
    # every layer at M = 1 in order, then every layer at M = 8
    assert calls[:len(layers)] == [(i, 1) for i in range(len(layers))]
    assert calls[len(layers):] == [(i, 8) for i in range(len(layers))]
    fr = {L["name"]: L["frac"] for L in layers}
    assert fr["L0.q"] == 0.1 and fr["L0.down"] == 0.2 and fr["L16.q"] == 0.7 and np.isclose(fr["L16.down"], 0.8)
    assert fr["L31.q"] == 0.1
    for L in layers:  # exact sparse-tile counts, weights drawn on the device later
        T = (L["N"] // 128) * (L["K"] // 128)
        assert int(L["bm"].sum()) == si.exact_sparse_count(T, L["frac"]) and "gen" in L and "w" not in L
    # distinct seeds per layer
    assert len({L["gen"] for L in layers}) == len(layers)


def test_llama3_qwen_layers_are_clustered_half_sparse():
    layers = bench.build_layers("llama3_qwen", only=["k", "v"])
    assert [L["name"] for L in layers] == ["llama3.k", "llama3.v", "qwen.k", "qwen.v"]
    for L in layers:
        T = (L["N"] // 128) * (L["K"] // 128)
        flat = L["bm"].ravel()
        on = np.flatnonzero(flat)
        assert len(on) == si.exact_sparse_count(T, 0.5) and on[-1] - on[0] + 1 == len(on)  # one contiguous run
        assert sorted(L["xs"]) == [1, 512]


def test_roofline_time_closed_forms():
    N, K, M = 256, 384, 100
    T = (N // 128) * (K // 128)
    dense = {"N": N, "K": K, "bm": np.zeros((2, 3), np.uint8)}
    sparse = {"N": N, "K": K, "bm": np.ones((2, 3), np.uint8)}
    assert np.isclose(bench.roof_seconds(dense, M, 1000.0, 2.0), 2 * M * N * K / 1e15)
    assert np.isclose(bench.roof_seconds(sparse, M, 1000.0, 2.0), 2 * M * N * K / 2e15)
    assert np.isclose(bench.roof_seconds(sparse, M, 1000.0, 1.5), 2 * M * N * K / 1.5e15)
    assert bench.stored_bytes(N, K, 0) == T * (32768 + 16)
    assert bench.stored_bytes(N, K, T) == T * (18432 + 16)


def test_bytes_block_throughput_and_segments():
    layers = [{"name": "a", "N": 128, "K": 128, "bm": np.zeros((1, 1), np.uint8), "frac": 0.0},
              {"name": "b", "N": 256, "K": 128, "bm": np.ones((2, 1), np.uint8), "frac": 1.0}]
    calls = [(0, 1), (1, 1), (0, 8), (1, 8)]
    by = [bench.call_bytes(layers[li], M) for li, M in calls]
    steps = 4
    t = _fake_t(ms_total=steps * 0.010)  # 10 us per step, no event split: proportional to bytes
    out = bench.bytes_block(_args(steps), "x", layers, calls, t, PK, 1, segments=[(0, 2), (2, 4)],
                            seg_names=["p1", "p8"])
    gbs = sum(by) / 1e9 / 10e-6
    assert np.isclose(out["value"], gbs, rtol=1e-3) and np.isclose(out["roofline"]["achieved"], gbs, rtol=1e-3)
    assert np.isclose(out["roofline"]["frac"], gbs / 6000.0, atol=1e-4)
    assert np.isclose(out["e2e"]["value"], gbs / 2, rtol=1e-3)
    assert set(out["per_segment"]) == {"p1", "p8"}
    # with an event split, segments take the measured shares of the event-free step time
    seg = np.tile([0.002, 0.006], (steps, 1))  # ms, scaled up to the 0.010 ms step
    out = bench.bytes_block(_args(steps), "x", layers, calls, _fake_t(steps * 0.010, seg), PK, 1,
                            segments=[(0, 2), (2, 4)], seg_names=["p1", "p8"])
    assert np.isclose(out["per_segment"]["p1"]["us"], 2.5) and np.isclose(out["per_segment"]["p8"]["us"], 7.5)


def test_flops_block_and_monotonic_sweep():
    layers = [{"name": "q", "N": 256, "K": 256, "bm": bm, "frac": f}
              for f, bm in ((0.0, np.zeros((2, 2), np.uint8)), (0.5, np.array([[1, 0], [0, 1]], np.uint8)),
                            (1.0, np.ones((2, 2), np.uint8)))]
    calls = [(0, 65536), (1, 65536), (2, 65536)]
    steps = 2
    seg = np.tile([0.004, 0.003, 0.002], (steps, 1))
    out, split = bench.flops_block(_args(steps), "p", layers, calls, _fake_t(steps * 0.009, seg), PK, 1,
                                   sparse_ratio=1.7)
    fl = 2 * 65536 * 256 * 256
    assert np.isclose(out["value"], 3 * fl / 1e12 / 9e-6, rtol=1e-3)
    r2 = sum(bench.roof_seconds(L, 65536, 1500.0, 2.0) for L in layers)
    assert np.isclose(out["roofline"]["frac"], r2 / 9e-6, atol=1e-4)
    rm = sum(bench.roof_seconds(L, 65536, 1500.0, 1.7) for L in layers)
    assert np.isclose(out["roofline"]["frac_measured_sparse_peak"], rm / 9e-6, atol=1e-4)
    # the tensor cores' own work: all-dense 4 tiles, half-sparse 3 tile-equivalents, all-sparse 2
    tile = 2 * 65536 * 128 * 128
    assert np.isclose(out["roofline"]["algorithmic_tflops"], (4 + 3 + 2) * tile / 1e12 / 9e-6, rtol=1e-3)
    assert np.isclose(out["per_call"]["q/f=1.0@M=65536"]["algorithmic_TFLOP/s"], 2 * tile / 1e12 / 2e-6, rtol=1e-2)
    sweep, mono = bench.sweep_summary(layers, calls, split)
    assert mono and sweep["q"]["speedup_vs_all_dense"] == [1.0, round(4 / 3, 3), 2.0]
    # a slower middle fraction breaks monotonicity
    sweep, mono = bench.sweep_summary(layers, calls, np.array([0.004, 0.005, 0.002]))
    assert not mono and not sweep["q"]["monotonic"]


def test_group_flops_block_over_segments():
    """Calls timed as group launches: the step's TFLOP/s and mixed-roofline
    fraction over all calls, and per segment (one launch) its own share."""
    layers = [{"name": "q", "N": 256, "K": 256, "bm": bm, "frac": f}
              for f, bm in ((0.0, np.zeros((2, 2), np.uint8)), (1.0, np.ones((2, 2), np.uint8)))]
    calls = [(0, 65536), (1, 65536), (0, 512), (1, 512)]
    steps = 2
    segs = [(0, 2), (2, 4)]
    seg = np.tile([0.006, 0.002], (steps, 1))  # ms per launch, the step 0.008 ms
    out = bench.group_flops_block(_args(steps), layers, calls, _fake_t(steps * 0.008, seg), PK, 1, segs,
                                  ["big", "small"], sparse_ratio=1.7)
    fl = np.array([2 * M * 256 * 256 for _, M in calls], dtype=np.float64)
    assert np.isclose(out["value"], fl.sum() / 1e12 / 8e-6, rtol=1e-3)
    r2 = [bench.roof_seconds(layers[li], M, 1500.0, 2.0) for li, M in calls]
    assert np.isclose(out["roofline"]["frac"], sum(r2) / 8e-6, atol=1e-4)
    rm = sum(bench.roof_seconds(layers[li], M, 1500.0, 1.7) for li, M in calls)
    assert np.isclose(out["roofline"]["frac_measured_sparse_peak"], rm / 8e-6, atol=1e-4)
    assert np.isclose(out["per_segment"]["big"]["us"], 6.0) and np.isclose(out["per_segment"]["small"]["us"], 2.0)
    assert np.isclose(out["per_segment"]["small"]["TFLOP/s"], fl[2:].sum() / 1e12 / 2e-6, rtol=1e-2)
    assert np.isclose(out["per_segment"]["big"]["roofline_frac"], (r2[0] + r2[1]) / 6e-6, atol=2e-3)
    # one segment: no per-segment split
    one = bench.group_flops_block(_args(steps), layers, calls, _fake_t(steps * 0.008, None), PK, 1, [(0, 4)], ["all"])
    assert "per_segment" not in one and np.isclose(one["value"], out["value"], rtol=1e-6)


def test_job_throughput_counts_every_rank():
    assert bench.job_throughput(2.0, 5, 4, 1000.0) == 2.0 * 5 * 4


@pytest.mark.parametrize("workload", ["all", "decode", "decode_fused", "prefill", "stack", "llama3_qwen"])
def test_run_ours_assembles_every_block_on_fake_timings(monkeypatch, workload):
    """The default run's JSON assembly (every block and mode) on CPU: GPU work is
    replaced by fakes that return fixed timings, so a missing or misnamed key in
    any block fails here rather than on the GPU machine."""
    import types

    import torch

    class FakePacked:
        def __init__(self, L):
            self.stored_bytes = bench.stored_bytes(L["N"], L["K"], int(L["bm"].sum()))

    def fake_time_calls(args, layers, packed, calls, dev, world, status, segments=None, chain=False, after=True,
                        gather=None, group=False):
        segs = segments or ([(0, len(calls))] if chain else [(j, j + 1) for j in range(len(calls))])
        return {"ms": 1.0 * args.steps, "e2e_ms": 2.0 * args.steps, "seg_ms": None, "clocks": {"sm_mhz": 1965.0},
                "h2d": 1, "d2h": 1, "launches": len(segs)}

    monkeypatch.setattr(bench, "pack_layers", lambda layers, dev, status: [FakePacked(L) for L in layers])
    monkeypatch.setattr(bench, "time_calls", fake_time_calls)
    monkeypatch.setattr(bench, "offline_steps", lambda layers, dev, pk: {})
    monkeypatch.setattr(bench, "mlp_steps", lambda dev, pk: {})
    monkeypatch.setattr(bench, "mma_rates", lambda dev: {"sparse_over_dense": 1.5})
    monkeypatch.setattr(bench, "build_layers", lambda w, *a: bench_small_layers(w))
    monkeypatch.setattr(torch.cuda, "set_device", lambda d: None)
    monkeypatch.setattr(torch.cuda, "synchronize", lambda: None)
    monkeypatch.setattr(torch.cuda, "empty_cache", lambda: None)
    import tile_sparse_gemm_b200 as tsg
    monkeypatch.setattr(tsg, "new_status", lambda dev=None: None)
    args = types.SimpleNamespace(steps=4, warmup=3, no_graph=False, layers=None, fracs=None, tokens=None,
                                 shard=False, workload=workload)
    out = bench.run_ours(args, 0, 1)
    for key in ("metric", "value", "unit", "ms_per_step", "roofline", "e2e", "clocks", "config", "gpu_launches"):
        assert key in out, key  # every workload alone gives a full line
    assert out["value"] > 0
    if workload != "all":
        return
    for key in ("metric", "value", "unit", "ms_per_step", "roofline", "e2e", "clocks", "config", "gpu_launches",
                "separate_calls", "chain_dependent", "prefill", "stack", "llama3_qwen", "mma_probe"):
        assert key in out, key
    assert out["config"]["blocks"] == list(bench.BLOCKS)
    assert out["prefill"]["roofline"]["frac_measured_sparse_peak"] > 0 and "sweep" in out["prefill"]
    for key in ("chain", "chain_independent"):
        assert "ms_per_pass" in out["stack"][key]
    assert set(out["llama3_qwen"]) >= {"M=1", "M=512"}
    assert out["llama3_qwen"]["M=1"]["chain_independent"]["value"] > 0
    assert out["llama3_qwen"]["M=512"]["group"]["value"] > 0 and "frac" in out["llama3_qwen"]["M=512"]["group"]["roofline"]
    assert set(out["prefill"]["group"]["per_segment"]) == {f"f={f}" for f in bench.FRACS}
    import json
    json.dumps(out)  # serialisable


@pytest.mark.parametrize("workload", ["decode", "prefill"])
def test_run_ours_sharded_blocks_on_fake_timings(monkeypatch, workload):
    """--shard with two ranks: each rank's block is its column-parallel shard
    plus one all-gather per step (the timer is faked); the line reports the
    whole job's throughput as strong scaling, balanced by bytes for decode and
    by tensor-core work for prefill."""
    import types

    import torch
    seen = {}

    class FakePacked:
        def __init__(self, L):
            self.stored_bytes = bench.stored_bytes(L["N"], L["K"], int(L["bm"].sum()))

    def fake_time_calls(args, layers, packed, calls, dev, world, status, segments=None, chain=False, after=True,
                        gather=None, group=False):
        seen["gather"], seen["N"] = gather, [L["N"] for L in layers]
        return {"ms": 1.0 * args.steps, "e2e_ms": 2.0 * args.steps, "seg_ms": None, "clocks": {"sm_mhz": 1965.0},
                "h2d": 1, "d2h": 1, "launches": 2}

    monkeypatch.setattr(bench, "pack_layers", lambda layers, dev, status: [FakePacked(L) for L in layers])
    monkeypatch.setattr(bench, "time_calls", fake_time_calls)
    monkeypatch.setattr(bench, "mma_rates", lambda dev: {"sparse_over_dense": 1.5})
    monkeypatch.setattr(bench, "build_layers", lambda w, *a: bench_small_layers(w, rows=6))
    monkeypatch.setattr(torch.cuda, "set_device", lambda d: None)
    monkeypatch.setattr(torch.cuda, "synchronize", lambda: None)
    monkeypatch.setattr(torch.cuda, "empty_cache", lambda: None)
    import tile_sparse_gemm_b200 as tsg
    monkeypatch.setattr(tsg, "new_status", lambda dev=None: None)
    args = types.SimpleNamespace(steps=4, warmup=3, no_graph=False, layers=None, fracs=None, tokens=None,
                                 shard=True, workload=workload)
    out = bench.run_ours(args, 0, 2)
    assert out["scaling"] == "strong" and "sharded" in out["metric"] and out["value"] > 0
    assert out["config"]["shard_balance"] == ("bytes" if workload == "decode" else "flops")
    assert seen["gather"] > 0 and all(n < 6 * 128 for n in seen["N"])  # rank 0 holds a part of every layer


def bench_small_layers(workload, rows=2):
    """Small stand-ins for each workload's layers (shapes, bitmaps and X only)."""
    rng = np.random.default_rng(0)

    def L(name, N, K, frac, ms, **kw):
        T = (N // 128) * (K // 128)
        bm = np.zeros(T, np.uint8)
        bm[:si.exact_sparse_count(T, frac)] = 1
        return dict(name=name, N=N, K=K, bm=bm.reshape(N // 128, K // 128), frac=frac,
                    xs={M: np.zeros((M, K), np.uint16) for M in ms}, **kw)
    if workload in ("decode", "decode_fused"):
        return [L(n, 128 * rows, 256, 0.5, (1, 4, 16)) for n in ("q", "gate")]
    if workload == "prefill":
        return [L(n, 128 * rows, 256, f, (2048,)) for n in ("q", "down") for f in bench.FRACS]
    if workload == "stack":
        return [L(f"L{i}.{n}", 256, 256, 0.1, (1, 8), proj=n) for i in range(2) for n in ("q", "down")]
    if workload == "llama3_qwen":
        return [L(n, 256, 128, 0.5, (1, 512)) for n in ("llama3.q", "qwen.k")]
    raise ValueError(workload)
