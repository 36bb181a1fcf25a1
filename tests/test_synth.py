"""The seeded input generators (synth/), checked on the CPU against what their published
definitions fix.  Both the CUDA path's tests and the oracle read these inputs, so a fault here
would not show as a parity failure; these checks pin the generators on their own.

  * SplitMix64 (Steele, Lea & Flood, OOPSLA 2014): the output function at state 0 gives the
    published first output 0xE220A8397B1DCDAF, and the words of one stream are the successive
    outputs of one SplitMix64 sequence (the stream's starting state is recovered from its first
    word by inverting the output function, which is a bijection of 64-bit words);
  * counter mode: a prefix of a longer draw equals a shorter draw;
  * Box-Muller normals and uniforms: sample moments within a few standard errors, ranges held;
  * bf16 storage: round to nearest even, checked on hand-made bit patterns.
"""
import numpy as np

import synth

M64 = (1 << 64) - 1
GAMMA = 0x9E3779B97F4A7C15
M1, M2 = 0xBF58476D1CE4E5B9, 0x94D049BB133111EB


def mix(z):
    """SplitMix64's output function on a 64-bit state (after the increment)."""
    z = ((z ^ (z >> 30)) * M1) & M64
    z = ((z ^ (z >> 27)) * M2) & M64
    return z ^ (z >> 31)


def unxorshift(y, s):
    """inverse of y = x ^ (x >> s) on 64-bit words"""
    x = y
    for _ in range(64 // s + 1):
        x = y ^ (x >> s)
    return x & M64


def unmix(z):
    z = unxorshift(z, 31)
    z = (z * pow(M2, -1, 1 << 64)) & M64
    z = unxorshift(z, 27)
    z = (z * pow(M1, -1, 1 << 64)) & M64
    return unxorshift(z, 30)


def test_splitmix64_known_answer_and_inverse():
    assert mix(GAMMA) == 0xE220A8397B1DCDAF
    rng = np.random.default_rng(0)
    for z in [0, 1, M64, GAMMA] + [int(v) for v in rng.integers(0, 1 << 63, 20)]:
        assert unmix(mix(z)) == z


def test_stream_words_are_one_splitmix64_sequence():
    for seed, tid in [(0, 1), (7, 1000 + 32 * 5 + 2), (123456789, 4)]:
        w = [int(v) for v in synth.uniform_u64(seed, tid, 64)]
        state = unmix(w[0])
        for i in range(1, 64):
            state = (state + GAMMA) & M64
            assert w[i] == mix(state)


def test_counter_mode_prefixes_agree():
    a = synth.normal_f32(3, 9, (1001,), 0.0, 1.0)
    b = synth.normal_f32(3, 9, (37,), 0.0, 1.0)
    assert np.array_equal(a[:37], b)               # b's last element is the first of a pair
    u = synth.uniform_u64(3, 9, 500)
    assert np.array_equal(u[:100], synth.uniform_u64(3, 9, 100))
    assert not np.array_equal(synth.uniform_u64(3, 10, 100), u[:100])
    assert not np.array_equal(synth.uniform_u64(4, 9, 100), u[:100])


def test_normal_and_uniform_moments():
    n = 1 << 20
    x = synth.normal_f32(1, 2, (n,), 0.5, 0.02).astype(np.float64)
    se = 0.02 / np.sqrt(n)
    assert abs(x.mean() - 0.5) < 5 * se
    assert abs(x.std() - 0.02) < 5 * 0.02 / np.sqrt(2 * n)
    z = (x - 0.5) / 0.02
    assert abs(np.mean(z ** 4) - 3.0) < 0.05                       # normal kurtosis
    assert abs(np.mean(np.abs(z) < 1.0) - 0.6826894921) < 0.003
    u = synth.uniform_f32(1, 3, (n,), -4.0, -2.0).astype(np.float64)
    assert u.min() >= -4.0 and u.max() < -2.0
    assert abs(u.mean() + 3.0) < 5 * (2.0 / np.sqrt(12 * n))
    assert abs(u.var() - 4.0 / 12) < 0.01
    k = synth.uniform_i32(1, 4, (n,), -127, 127)
    assert k.min() == -127 and k.max() == 127
    counts = np.bincount(k + 127, minlength=255)
    assert counts.min() > 0.8 * n / 255 and counts.max() < 1.2 * n / 255


def test_bf16_storage_rounds_to_nearest_even():
    def f(bits):
        return np.array([bits], np.uint32).view(np.float32)
    # 1.0 + half an ulp of bf16 (a tie) rounds to even (1.0); just above the tie rounds up
    assert synth.f32_to_bf16(f(0x3F808000))[0] == 0x3F80
    assert synth.f32_to_bf16(f(0x3F808001))[0] == 0x3F81
    # an odd bf16 neighbour: the tie rounds up to the even one
    assert synth.f32_to_bf16(f(0x3F818000))[0] == 0x3F82
    assert synth.f32_to_bf16(f(0xBF817FFF))[0] == 0xBF81
    v = synth.normal_f32(5, 5, (4096,))
    back = synth.bf16_to_f32(synth.f32_to_bf16(v))
    assert np.all(np.abs(back - v) <= np.abs(v) * 2.0 ** -8)
