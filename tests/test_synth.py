"""The seeded input generator: reproducible, thread-count independent, right laws."""
import os
import subprocess
import sys

import numpy as np

import synth


def test_same_seed_same_bits_and_prefix_consistent():
    a = synth.normal_bf16(9, 1, (64, 256), 1.0)
    b = synth.normal_bf16(9, 1, (128, 256), 1.0)
    assert np.array_equal(a, b[:64])
    assert not np.array_equal(a, synth.normal_bf16(10, 1, (64, 256), 1.0))
    assert not np.array_equal(a, synth.normal_bf16(9, 2, (64, 256), 1.0))


def test_thread_count_does_not_change_values():
    code = ("import synth, numpy as np, sys; "
            "a = synth.normal_bf16(4, 10, (300, 512), 0.5); c, s = synth.fp8_blocks(4, 10, 2, 128, 256, 0.5); "
            "sys.stdout.write(str(int(a.astype(np.uint64).sum())) + ' ' + str(int(c.astype(np.uint64).sum())) "
            "+ ' ' + repr(float(s.sum())))")
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    outs = []
    for n in ("1", "4"):
        env = dict(os.environ, OMP_NUM_THREADS=n, PYTHONPATH=root)
        outs.append(subprocess.check_output([sys.executable, "-c", code], env=env, cwd=root).decode())
    assert outs[0] == outs[1]


def test_normal_moments():
    v = synth.bf16_to_f32(synth.normal_bf16(1, 1, (1 << 20,), 0.25)).astype(np.float64)
    assert abs(v.mean()) < 2e-3 and abs(v.std() - 0.25) < 1e-3


def test_fp8_blocks_are_the_quantised_bf16_draws():
    G, R, C, std = 2, 256, 384, 1 / 16
    codes, scales = synth.fp8_blocks(8, 10, G, R, C, std)
    ref = synth.bf16_to_f32(synth.normal_bf16(8, 10, (G, R, C), std)).astype(np.float64)
    vals = synth.e4m3_value_table().astype(np.float64)[codes]
    blk = ref.reshape(G, R // 128, 128, C // 128, 128)
    amax = np.abs(blk).max(axis=(2, 4))
    np.testing.assert_array_equal(scales, (amax.astype(np.float32) / np.float32(448.0)))
    deq = vals * np.repeat(np.repeat(scales, 128, axis=1), 128, axis=2)
    assert np.abs(vals).reshape(G, R // 128, 128, C // 128, 128).max(axis=(2, 4)).min() == 448.0
    rel = np.abs(deq - ref) / np.abs(ref).clip(1e-30)
    normal = np.abs(vals) >= 2 ** -6
    assert rel[normal].max() <= 2 ** -4 + 1e-6


def test_zipf_bias_is_a_ranking():
    b = synth.zipf_bias(3, 352)
    r = np.exp(-b / (synth.ZIPF_S * synth.ZIPF_ALPHA))
    assert np.allclose(np.sort(r), np.arange(1, 353), rtol=1e-5)
