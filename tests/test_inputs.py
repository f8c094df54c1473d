"""The seeded synthetic inputs (shared by the oracle and the GPU path) follow
their stated recipe: seeds, distributions, exact sparse-tile counts, banded
placement and the 32-layer stack's fraction schedule.  CPU only."""
import numpy as np
import pytest

import synth_inputs as si


def test_seed_recipe_and_streams_are_distinct():
    a = si.rng(2, 3, si.STREAM_W).standard_normal(8)
    b = np.random.Generator(np.random.PCG64(20250927 + 1000 * 2 + 10 * 3 + 1)).standard_normal(8)
    assert np.array_equal(a, b)
    draws = {s: si.rng(2, 3, s).standard_normal(4).tobytes() for s in range(5)}
    assert len(set(draws.values())) == 5
    assert np.array_equal(si.gen_x(4, 256, 1, 2), si.gen_x(4, 256, 1, 2))  # deterministic


def test_weight_and_activation_distributions():
    w = si.bf16_bits_to_f32(si.gen_w(512, 1024, 2, 0)).astype(np.float64)
    x = si.bf16_bits_to_f32(si.gen_x(64, 4096, 2, 0)).astype(np.float64)
    assert abs(w.mean()) < 1e-3 and abs(w.std() - 0.02) < 2e-4
    assert abs(x.mean()) < 2e-2 and abs(x.std() - 1.0) < 1e-2


@pytest.mark.parametrize("frac", [0.0, 0.25, 0.5, 0.75, 1.0])
def test_exact_and_clustered_tile_counts(frac):
    N, K = 1024, 1536
    T = (N // 128) * (K // 128)
    want = int(np.floor(frac * T + 0.5))
    assert int(si.tiles_exact(N, K, frac, 2, 0).sum()) == want
    band = si.tiles_clustered(N, K, frac, 5, 0).reshape(-1)
    assert int(band.sum()) == want
    if want:
        idx = np.flatnonzero(band)
        assert idx[-1] - idx[0] + 1 == want  # one contiguous run in row-major tile order


@pytest.mark.parametrize("b", [4, 16, 64, 128])
@pytest.mark.parametrize("clustered", [False, True])
def test_mask_tiles_counts_placement_and_choice_logits(b, clustered):
    N, K = 512, 768
    kinds = si.mask_tiles(N, K, b, 0.5, clustered, 3, b)
    T = (N // b) * (K // b)
    assert kinds.shape == (N // b, K // b)
    assert int(kinds.sum()) == int(np.floor(0.5 * T + 0.5))
    if clustered:
        idx = np.flatnonzero(kinds.reshape(-1))
        assert idx[-1] - idx[0] + 1 == idx.size
    logits = si.choice_logits(kinds)
    assert np.array_equal(np.argmax(logits, axis=-1), kinds)  # no ties: the argmax is the kind


def test_stack_fraction_schedule():
    attn, mlp = ("q", "k", "v", "o"), ("gate", "up", "down")
    for layer in range(32):
        edge = layer < 4 or layer >= 28
        for p in attn:
            assert si.stack_fraction(layer, p) == (0.1 if edge else 0.7)
        for p in mlp:
            assert si.stack_fraction(layer, p) == pytest.approx(0.2 if edge else 0.8)


def test_workload_shapes_are_tile_multiples():
    for table in (si.LLAMA2_7B, si.LLAMA3_8B, si.QWEN25_05B, si.GEMMA3_1B):
        for _, N, K in table:
            assert N % 128 == 0 and K % 128 == 0
    assert dict((n, (N, K)) for n, N, K in si.LLAMA2_7B) == {
        "q": (4096, 4096), "k": (4096, 4096), "v": (4096, 4096), "o": (4096, 4096),
        "gate": (11008, 4096), "up": (11008, 4096), "down": (4096, 11008)}


def test_device_generators_match_the_host_recipe():
    """The torch form of the magnitude top-2 choice (used for workloads drawn on
    the device) equals the numpy form, ties and signed zeros included; the torch
    weight draw is seeded (repeatable) with the recipe's distribution."""
    import torch
    rng = np.random.default_rng(5)
    w = si.f32_to_bf16_bits(rng.standard_normal((64, 256)).astype(np.float32) * 0.02)
    w[0, :8] = [0x3F80, 0xBF80, 0x3F80, 0x0000, 0x8000, 0x0000, 0x8000, 0x0000]  # ties, +0 / -0
    w[1, :4] = 0x3F80
    wt = torch.from_numpy(w.view(np.int16)).view(torch.bfloat16)
    assert np.array_equal(si.patterns_top2_torch(wt).numpy(), si.patterns_top2(w))
    a = si.gen_w_device(256, 512, 4, 3, "cpu")
    b = si.gen_w_device(256, 512, 4, 3, "cpu")
    assert a.dtype == torch.bfloat16 and torch.equal(a.view(torch.int16), b.view(torch.int16))
    assert not torch.equal(a.view(torch.int16), si.gen_w_device(256, 512, 4, 4, "cpu").view(torch.int16))
    std = float(a.float().std())
    assert 0.019 < std < 0.021 and abs(float(a.float().mean())) < 1e-3
