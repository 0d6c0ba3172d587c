"""Pins for the seeded input generators (host twin) and, on a GPU, twin identity."""
import math
import os

import numpy as np
import pytest

from sidgen import host

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rows(name):
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                yield line.split()


def test_philox_known_answers():
    for cols in _rows("philox4x32_10_kat.txt"):
        v = [int(x, 16) for x in cols]
        seed = v[4] | (v[5] << 32)
        out = host.philox4x32_10(v[0], v[1], v[2], v[3], seed)
        assert [int(x) for x in out] == v[6:10]


def test_splitmix64_reference_outputs():
    for seed, idx, val in _rows("splitmix64_ref.txt"):
        got = host.splitmix64_stream(int(seed), int(idx), 1)[0]
        assert int(got) == int(val)


def test_normal_draws_moments_and_bounds():
    c = np.arange(200_000, dtype=np.uint64)
    x = host.normal_from_counters(7, c, 0, 0, 0, 3.0).astype(np.float64)
    assert abs(x.mean()) < 0.03
    assert abs(x.std() - 3.0) < 0.02
    # Irwin-Hall of eight terms is bounded at sqrt(3*8) = 4.899 sigma.
    assert np.abs(x).max() <= 3.0 * math.sqrt(24.0) + 1e-4
    # Excess kurtosis of the sum of 8 uniforms is -1.2/8.
    k = ((x - x.mean()) ** 4).mean() / x.var() ** 2 - 3.0
    assert abs(k + 0.15) < 0.05


def test_bf16_rounding_is_nearest_even():
    # 1 + 2^-8 is exactly halfway between bf16 1.0 and 1 + 2^-7: ties to even -> 1.0.
    vals = np.array([1.0, 1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, -2.5, 0.0], dtype=np.float32)
    bits = host.f32_to_bf16_bits(vals)
    back = host.bf16_bits_to_f32(bits)
    assert back.tolist() == [1.0, 1.0, 1.0 + 2 * 2.0 ** -7, -2.5, 0.0]


def test_prefix_hash_chains():
    pre = np.array([[3, 5, 7], [3, 5, 8]])
    h = host.prefix_hashes(pre)
    manual = host.child_hash(host.child_hash(host.child_hash(host.root_hash(), 1, 3), 2, 5), 3, 7)
    assert int(h[0]) == int(manual)
    assert h[0] != h[1]
    empty = np.zeros((3, 0), dtype=np.int64)
    assert int(host.prefix_hashes(empty)[0]) == int(host.root_hash(0))
    roots = host.prefix_hashes(empty, np.array([0, 1, 2]))
    assert len({int(x) for x in roots}) == 3          # requests start from distinct roots
    assert int(roots[2]) == int(host.splitmix64_mix(np.uint64(host.PREFIX_HASH_SEED ^ 2)))
    h1 = host.prefix_hashes(pre, np.array([1, 1]))
    assert int(h1[0]) == int(host.child_hash(host.child_hash(host.child_hash(
        host.root_hash(1), 1, 3), 2, 5), 3, 7))


def test_catalog_draw_distinct_and_in_range():
    cat = host.draw_catalog(1001, 2000, [32, 32, 32])
    assert cat.shape == (2000, 3)
    assert len({tuple(r) for r in cat.tolist()}) == 2000
    assert cat.min() >= 0 and cat.max() < 32
    # Reproducible.
    assert np.array_equal(cat, host.draw_catalog(1001, 2000, [32, 32, 32]))


def test_zipf_level_frequencies():
    V, s = 64, 1.1
    x = host.splitmix64_stream(99, 0, 400_000)
    codes = host._zipf_codes(x, host._zipf_cdf(V, s))
    freq = np.bincount(codes, minlength=V) / codes.shape[0]
    pmf = np.arange(1, V + 1, dtype=np.float64) ** -s
    pmf /= pmf.sum()
    assert np.abs(freq - pmf).max() < 3e-3
    assert freq[0] > freq[1] > freq[10]


def test_catalog_rejects_impossible_size():
    with pytest.raises(ValueError):
        host.draw_catalog(1, 10, [3, 3])


@pytest.mark.gpu
def test_device_twin_bit_identical():
    import torch
    from sidgen import device
    device.build()
    rng = np.random.default_rng(5)
    n = 1 << 20
    ctr = rng.integers(0, 2**32, size=(n, 4), dtype=np.uint64)
    seed = 0x1234_5678_9ABC_DEF0
    ref = np.stack(host.philox4x32_10(ctr[:, 0], ctr[:, 1], ctr[:, 2], ctr[:, 3], seed), axis=1)
    d_ctr = torch.from_numpy(ctr.astype(np.uint32).view(np.int32)).cuda()
    d_out = torch.empty_like(d_ctr)
    device.philox(seed, d_ctr, d_out)
    got = d_out.cpu().numpy().view(np.uint32)
    assert np.array_equal(got, ref.astype(np.uint32))

    # Logits rows, fp32 and bf16, with a padded leading dimension.
    hashes = host.prefix_hashes(rng.integers(0, 100, size=(300, 2)))
    for dt, tdt in (("f32", torch.float32), ("bf16", torch.bfloat16)):
        ref = host.row_logits(42, hashes, 777, 2.5, dtype=dt)
        out = torch.zeros((300, 784), dtype=tdt, device="cuda")
        device.row_logits(42, torch.from_numpy(hashes.view(np.int64)).cuda(), 777, 2.5, out)
        got = out[:, :777].cpu()
        got = got.view(torch.int16).numpy().view(np.uint16) if dt == "bf16" else got.numpy()
        assert np.array_equal(got, ref)

    # Score tables, weights, hidden states.
    ref = host.table_logits(9, 3, 4, 256, 1.5)
    out = torch.empty((3, 4, 256), dtype=torch.float32, device="cuda")
    device.table(9, 3, 4, 256, 1.5, out)
    assert np.array_equal(out.cpu().numpy(), ref)
    ref = host.weight_matrix(11, 100, 64, 0.02)
    out = torch.empty((100, 64), dtype=torch.int16, device="cuda")
    device.weight(11, 100, 64, 0.02, out)
    assert np.array_equal(out.cpu().numpy().view(np.uint16), ref)
    ref = host.hidden_states(12, hashes[:50], 64, 1.0)
    out = torch.empty((50, 64), dtype=torch.int16, device="cuda")
    device.hidden(12, torch.from_numpy(hashes[:50].view(np.int64)).cuda(), 64, 1.0, out)
    assert np.array_equal(out.cpu().numpy().view(np.uint16), ref)
