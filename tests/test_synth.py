"""The synthetic-input module's own claims: its fp32 -> bf16 rounding is
round-to-nearest-even (torch's bfloat16 cast decides), large draws made in
blocks equal one draw of the whole shape, and every workload's inputs are
reproducible from its seed."""

import numpy as np
import torch

from fp8_transformer_block_b200 import synth


def test_bf16_rounding_is_nearest_even():
    rng = np.random.default_rng(0)
    u = rng.integers(0, 2 ** 32, size=400_000, dtype=np.uint64).astype(np.uint32)
    u = u[((u >> 23) & 0xFF) != 0xFF]                       # finite values
    ties = (u & np.uint32(0xFFFF0000)) | np.uint32(0x8000)   # exact midpoints
    edge = np.array([0.0, -0.0, 1.0, -1.0, 3.3895314e38, -3.3895314e38, 1e-40, 2.0 ** -133],
                    np.float32)
    for x in (u.view(np.float32), ties.view(np.float32), edge):
        want = torch.from_numpy(x.copy()).to(torch.bfloat16).view(torch.int16).numpy()
        assert np.array_equal(synth.bf16_bits(x), want.view(np.uint16))


def test_block_draws_equal_one_draw():
    shape = (6000, 3000)  # above the block size: drawn in blocks of rows
    a = synth.normal_bf16(np.random.Generator(np.random.PCG64(11)), shape, 0.02)
    ref = synth.bf16_bits(np.random.Generator(np.random.PCG64(11))
                          .standard_normal(size=shape, dtype=np.float32) * np.float32(0.02))
    assert np.array_equal(a, ref)


def test_inputs_reproduce_from_the_seed():
    w = synth.WORKLOADS["vla_action_expert"]
    a = synth.adarms_inputs(w.rows, w.D, w.seed, outliers=True)
    b = synth.adarms_inputs(w.rows, w.D, w.seed, outliers=True)
    for k in a:
        assert np.array_equal(a[k], b[k])
    m1 = synth.modulation_inputs(1, 64, 3, 5)
    m2 = synth.modulation_inputs(1, 64, 3, 5)
    assert all(np.array_equal(m1[k], m2[k]) for k in m1)
    assert not np.array_equal(m1["w"], synth.modulation_inputs(1, 64, 3, 6)["w"])
