"""The seeded input generators: the host (numpy) generator the parity tests
use and the device (torch) generator the bench draws its large inputs from
follow one recipe, so they agree: the 64-bit counter stream and the uniforms
bit for bit, the normals to a few ulp, the bf16 inputs exactly on these
cases.  The stream itself is checked against splitmix64's definition."""
import numpy as np
import pytest

import synth
from synth import torch_latents as TL
from synth.video_latents import round_to

torch = pytest.importorskip("torch")


def _mix64_reference(x: int) -> int:
    """splitmix64's output function written out with Python integers."""
    m = (1 << 64) - 1
    z = x & m
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & m
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & m
    return z ^ (z >> 31)


def test_stream_follows_the_definition():
    seed, off = 0x1234_5678_9ABC, 5
    z = synth.splitmix64_stream(seed, 64, offset=off)
    for i in range(64):
        assert int(z[i]) == _mix64_reference(seed + (off + i + 1) * 0x9E3779B97F4A7C15)


def test_chunked_host_stream_equals_one_pass():
    n = (1 << 22) + 12345                  # more than one chunk
    u = synth.uniform01(77, n)
    z = synth.splitmix64_stream(77, n)
    ref = ((z >> np.uint64(11)).astype(np.float64) + 1.0) * 2.0 ** -53
    assert np.array_equal(u, ref)


def test_device_generator_matches_host_generator():
    z_np = synth.splitmix64_stream(12345, 3000, offset=7)
    z_t = TL.splitmix64_stream(12345, 3000, offset=7, device="cpu")
    assert np.array_equal(z_np.view(np.int64), z_t.numpy())
    assert np.array_equal(synth.uniform01(99, 5000), TL.uniform01(99, 5000, device="cpu").numpy())
    a = synth.standard_normal(99, 20000)
    b = TL.standard_normal(99, 20000, device="cpu").numpy()
    assert np.max(np.abs(a - b)) <= 1e-14
    for head_gain in (False, True):
        hq = synth.make_qkv(5, 4, 3, 9, 16, 3, 64, head_gain=head_gain)
        tq = TL.make_qkv(5, 4, 3, 9, 16, 3, 64, head_gain=head_gain, device="cpu")
        for x, y in zip(hq, tq):
            assert np.array_equal(round_to(x, "bf16"), y.float().numpy().astype(np.float64))
    d = TL.make_dout(5, 4, 432, 3, 64, device="cpu").float().numpy().astype(np.float64)
    assert np.array_equal(round_to(synth.make_dout(5, 4, 432, 3, 64), "bf16"), d)
