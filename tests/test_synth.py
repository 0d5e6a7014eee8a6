"""The seeded generator: numpy path pinned to a pure-int SplitMix64, plus the
workload shapes and planted structure."""
import numpy as np

import synth


def _splitmix_ref(seed, tid, i):
    M = (1 << 64) - 1
    def mix(z):
        z &= M
        z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & M
        z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & M
        return z ^ (z >> 31)
    key = mix(seed * 0x9E3779B97F4A7C15 + tid)
    return mix(key + (i + 1) * 0x9E3779B97F4A7C15)


def test_hash_matches_reference_splitmix():
    idx = [0, 1, 2, 1000, 2**33 + 5]
    got = synth.hash_at(1237, 5, idx)
    for i, h in zip(idx, got):
        assert int(h) == _splitmix_ref(1237, 5, i)


def test_normal_is_irwin_hall_and_moments():
    h = _splitmix_ref(1, 2, 7)
    s = sum((h >> (16 * j)) & 0xFFFF for j in range(4))
    want = np.float32(s - 131070) * synth.IH_SCALE
    assert synth.normal_at(1, 2, [7])[0] == want
    x = synth.normal_at(3, 4, np.arange(200000)).astype(np.float64)
    assert abs(x.mean()) < 0.01 and abs(x.std() - 1) < 0.01
    assert x.max() <= 3.4642 and x.min() >= -3.4642


def test_bf16_rounding_nearest_even():
    vals = np.array([1.0, 1.0 + 2**-8, 1.0 + 3 * 2**-8, -2.5, 3.0e-3], np.float32)
    bits = synth.f32_to_bf16_bits(vals)
    back = synth.bf16_bits_to_f32(bits)
    assert back[0] == 1.0 and back[1] == 1.0 and back[2] == 1.0 + 2**-6 and back[3] == -2.5
    assert abs(back[4] - 3.0e-3) <= 2**-8 * 3.0e-3


def test_workload_shapes():
    c3 = synth.workload("c3")
    assert c3.B == 4 and c3.S_max == 131072 and c3.L == 24 and len(c3.groups) == 1
    c2 = synth.workload("c2")
    assert [list(g) for g in c2.groups] == [list(range(4 * i, 4 * i + 4)) for i in range(3)]
    c5 = synth.workload("c5")
    assert c5.B == 32 and all(8192 <= s <= 131072 for s in c5.seq_lens) and len(c5.groups) == 12
    assert len(set(c5.seq_lens)) > 20
    c4 = synth.workload("c4")
    regs = c4.regions()
    assert len(regs) == 16 and all(r % 64 == 0 and r + 256 <= c4.S - c4.chunk for r in regs)


def test_sampled_rows_equal_full_materialisation():
    c1 = synth.workload("c1")
    KI = c1.KI_full(0)
    rows = [0, 17, 4095] + [t for (_, t, _, _) in c1.planted(0)][:3]
    assert np.array_equal(c1.KI_rows(0, 0, rows), KI[rows])
    K = c1.KV_full(0, "K").reshape(c1.Hkv, c1.S_max, c1.d)
    assert np.array_equal(c1.KV_rows(0, 0, 0, rows, "K"), K[0, rows])


def test_q_autoregressive_correlation():
    c3 = synth.workload("c3")
    Q = synth.bf16_bits_to_f32(c3.Q()).astype(np.float64)
    r = np.corrcoef(Q[0].ravel(), Q[1].ravel())[0, 1]
    assert abs(r - 0.9) < 0.01
