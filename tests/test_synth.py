"""Pins for the shared input generator (no GPU)."""
import math

import numpy as np
import torch

import synth


def test_splitmix64_reference_outputs():
    """First outputs of splitmix64 seeded with 0 (Steele, Lea, Flood 2014;
    the published reference implementation's stream)."""
    L = synth.lib()
    assert [L.synth_splitmix64(0, i) for i in range(3)] == [
        0xE220A8397B1DCDAF, 0x6E789E6AA1B965F4, 0x06C45D188009454F]


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(100000).astype(np.float32) * 10 ** rng.uniform(-5, 5, 100000),
                        np.array([0.0, -0.0, 1.0, 1.00390625, 1.01171875], dtype=np.float32)]).astype(np.float32)
    ours = synth.f32_to_bf16(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(ours, ref)
    L = synth.lib()
    assert all(L.synth_bf16_rne(float(a)) == b for a, b in zip(x[:2000], ref[:2000]))


def test_generator_statistics_and_layout():
    w = synth.Workload("t", [(2, 8, 8), (1, 4, 5)], H=3, D=64, seed=1, amp=3.0)
    q, k, v = synth.generate(w, nthreads=3)
    assert q.shape == (148, 3, 64)
    vf = synth.bf16_to_f32(v)
    assert abs(vf.mean()) < 0.05 and abs(vf.std() - 1.0) < 0.05
    # Q - K has no positional part: variance 2
    dq = synth.bf16_to_f32(q).astype(np.float64) - synth.bf16_to_f32(k)
    assert abs(dq.var() - 2.0) < 0.1
    # positional code: token 0 of each sequence sits at (0,0,0): sin dims 0, cos dims 1
    L = synth.lib()
    pe0 = np.array([L.synth_pe(64, 0, 0, 0, d) for d in range(64)])
    assert np.allclose(pe0[0::2], 0) and np.allclose(pe0[1::2], 1)
    # same seed, same values; drawing a slice alone gives the same elements
    q2, _, _ = synth.generate(w, nthreads=1, tensors=("q",))
    np.testing.assert_array_equal(q, q2)
    # x position of the last token of sequence 0 is 7, y is 7, t is 1 (dims d_t=24, d_y=d_x=20)
    assert math.isclose(L.synth_pe(64, 1, 7, 7, 44), math.sin(7.0))
