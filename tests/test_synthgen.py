"""Pins of the seeded input generator (shared by both harnesses, holds no step arithmetic)."""
import bisect
import math

import numpy as np

import synthgen


def test_philox_known_answers():
    # Known-answer vectors of Philox4x32-10 published with the generator's reference
    # implementation (Random123, Salmon et al., SC'11).
    assert synthgen.philox([0, 0, 0, 0], [0, 0]) == [0x6627E8D5, 0xE169C58D, 0xBC57AC4C, 0x9B00DBD8]
    assert synthgen.philox([0xFFFFFFFF] * 4, [0xFFFFFFFF] * 2) == [
        0x408F276D, 0x41C83B0E, 0xA20BC7C6, 0x6D5451FD]
    assert synthgen.philox([0x243F6A88, 0x85A308D3, 0x13198A2E, 0x03707344],
                           [0xA4093822, 0x299F31D0]) == [0xD16CFE09, 0x94FDCCEB, 0x5001E420, 0x24126EA1]


def test_irwin_hall_moments():
    x = synthgen.normal_host(0, 1 << 20, seed=0, stream=1, step=1, sigma=1.0)
    assert abs(x.mean()) < 5e-3
    assert abs(x.var() - 1.0) < 5e-3
    assert np.abs(x).max() <= 2.0 * math.sqrt(3.0)
    # Irwin-Hall(4) kurtosis: 3 - 6/(5*4) = 2.7 (a normal has 3)
    kurt = np.mean(x ** 4) / np.mean(x ** 2) ** 2
    assert abs(kurt - 2.7) < 0.02


def _all_finite_bf16_values():
    bits = np.arange(0x8000, dtype=np.uint32)
    f = (bits << 16).view(np.float32)
    f = f[np.isfinite(f)].astype(np.float64)
    return np.unique(np.concatenate([-f, f]))


def _nearest_even_bf16(x, grid):
    """Brute force: nearest finite bf16 value, ties to the even encoding; inf past max + half ulp."""
    if math.isnan(x):
        return None
    maxf = grid[-1]
    half_ulp_top = (maxf - grid[-2]) / 2
    if x >= maxf + half_ulp_top:
        return math.inf
    if x <= -maxf - half_ulp_top:
        return -math.inf
    i = bisect.bisect_left(grid, x)
    cands = [grid[j] for j in (i - 1, i) if 0 <= j < len(grid)]
    best = min(cands, key=lambda c: abs(c - x))
    ties = [c for c in cands if abs(c - x) == abs(best - x)]
    if len(ties) == 2:
        enc = [int(np.float32(c).view(np.uint32) >> 16) for c in ties]
        best = ties[0] if enc[0] % 2 == 0 else ties[1]
    return best


def test_double_to_bf16_matches_brute_force():
    grid = list(_all_finite_bf16_values())
    rng = np.random.default_rng(1)
    xs = list(rng.normal(0, 1e-3, 3000)) + list(rng.normal(0, 1e3, 500))
    # exact ties and near-ties between neighbours, subnormals, overflow edge
    for a, b in zip(grid[1000:1400], grid[1001:1401]):
        mid = (a + b) / 2
        xs += [mid, np.nextafter(mid, -np.inf), np.nextafter(mid, np.inf)]
    xs += [0.0, -0.0, 1e-45, 9.2e-41, -9.2e-41, 3.3895313892515355e38, 3.39e38, 1e300]
    got = synthgen.round_double_to_half(np.array(xs), synthgen.BF16)
    for x, g in zip(xs, got):
        ref = _nearest_even_bf16(x, grid)
        val = float((np.uint32(g) << np.uint32(16)).view(np.float32))
        assert val == ref or (val == 0 and ref == 0), (x, hex(g), ref)


def test_double_to_fp16_matches_numpy():
    rng = np.random.default_rng(2)
    xs = np.concatenate([rng.normal(0, 1e-3, 20000) * 65536, rng.normal(0, 1e-4, 20000),
                         rng.normal(0, 3e4, 5000), [65504.0, 65519.99, 65520.0, 7e4, 6e-8,
                                                    2.98e-8, 2.9802322387695312e-08, -0.0]])
    # exact midpoints of neighbouring fp16 values (ties to even)
    h = np.arange(0, 0x7BFF, 7, dtype=np.uint16).view(np.float16).astype(np.float64)
    mids = (h[:-1] + np.nextafter(h[:-1].astype(np.float16), np.float16(np.inf)).astype(np.float64)) / 2
    xs = np.concatenate([xs, mids, -mids])
    got = synthgen.round_double_to_half(xs, synthgen.FP16)
    ref = xs.astype(np.float16).view(np.uint16)
    assert np.array_equal(got, ref)


def test_gradient_recipe_properties():
    n = 1 << 16
    g = synthgen.grads_host(0, n, seed=0, replica=0, slot=1, sigma=1e-3, spike_frac=0.0,
                            scale=1.0, dtype=synthgen.BF16)
    f = (g.astype(np.uint32) << 16).view(np.float32)
    assert abs(f.std() - 1e-3) < 2e-5
    # x8 spikes on ~0.1% of elements, exact in bf16
    gs = synthgen.grads_host(0, n, seed=0, replica=0, slot=1, sigma=1e-3, spike_frac=0.001,
                             scale=1.0, dtype=synthgen.BF16)
    fs = (gs.astype(np.uint32) << 16).view(np.float32)
    spiked = fs != f
    assert 20 < spiked.sum() < 120
    assert np.array_equal(fs[spiked], f[spiked] * 8)
    # loss scale 2^16 in fp16 is an exact power-of-two shift of the unscaled draw
    h1 = synthgen.grads_host(0, n, 0, 0, 1, 1e-3, 0.0, 65536.0, synthgen.FP16)
    x = synthgen.normal_host(0, n, 0, synthgen.STREAM_GRAD + 0, 1, 1e-3) * 65536.0
    assert np.array_equal(h1, x.astype(np.float16).view(np.uint16))
    # replicas and slots are different streams
    g2 = synthgen.grads_host(0, n, 0, 1, 1, 1e-3, 0.0, 1.0, synthgen.BF16)
    g3 = synthgen.grads_host(0, n, 0, 0, 2, 1e-3, 0.0, 1.0, synthgen.BF16)
    assert (g2 != g).mean() > 0.9 and (g3 != g).mean() > 0.9
    # index-list fill agrees with the range fill
    j = np.array([0, 5, 777, n - 1], np.uint64)
    assert np.array_equal(synthgen.grads_at_host(j, 0, 0, 1, 1e-3, 0.001, 1.0, synthgen.BF16),
                          gs[j.astype(np.int64)])


def test_workload_sizes():
    # parameter counts of the tensor lists (closed forms from the shapes)
    assert synthgen.workload("tiny").n == 1024 * 1024
    enc = synthgen.workload("enc")
    d, ff = 4096, 2048
    assert enc.n == 3 * d * d + 3 * d + d * d + d + ff * d + ff + d * ff + d + 4 * d == 83_924_992
    assert len(enc.tensors) == 12
    gpt2 = synthgen.workload("gpt2")
    assert gpt2.n == 354_823_168 and len(gpt2.tensors) == 292
    llama = synthgen.workload("llama7b")
    assert llama.n == 6_738_415_616 and len(llama.tensors) == 291


def test_inf_sites_are_seeded_and_in_range():
    enc = synthgen.workload("enc")
    s3 = enc.inf_sites_at(3)
    assert len(s3) == 5 and s3 == enc.inf_sites_at(3)
    assert all(0 <= i < enc.n and 0 <= r < enc.world for i, r in s3)
    assert enc.inf_sites_at(1) == []
    assert s3 != enc.inf_sites_at(7)
