"""CPU checks of the seeded input generator (host half)."""
import math

import numpy as np

import synth

MASK64 = (1 << 64) - 1


def _splitmix64_outputs(state, n):
    """SplitMix64 written out in plain Python from its published definition."""
    out = []
    for _ in range(n):
        state = (state + 0x9E3779B97F4A7C15) & MASK64
        z = state
        z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & MASK64
        z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & MASK64
        out.append(z ^ (z >> 31))
    return out


def test_splitmix64_published_vector():
    # reference output of splitmix64 seeded with 1234567 (Vigna's test sequence)
    want = [6457827717110365317, 3203168211198807973, 9817491932198370423,
            4593380528125082431, 16408922859458223821]
    lib = synth.host_lib()
    got = [lib.synth_splitmix64_at(1234567, c) for c in range(1, 6)]
    assert got == want
    assert _splitmix64_outputs(1234567, 5) == want


def _mix64(v):
    """SplitMix64's output function: the first output of a stream whose state is v - G."""
    return _splitmix64_outputs((v - 0x9E3779B97F4A7C15) & MASK64, 1)[0]


def _element_python(seed, tid, i, sigma, bf16=True):
    """One generator element, from the definition in synth_def.h, in plain Python."""
    key = _mix64(seed ^ _mix64((tid * 0x9E3779B97F4A7C15) & MASK64))
    words = _splitmix64_outputs(key, 3 * i + 3)[3 * i:3 * i + 3]
    s = sum((w >> (16 * q)) & 0xFFFF for w in words for q in range(4))
    z = np.float32((s - 393210) / 65536.0)  # exact in fp32
    v = np.float32(z * np.float32(sigma))  # one fp32 multiply
    if not bf16:
        return v
    u = int(np.array([v], dtype=np.float32).view(np.uint32)[0])
    u = (u + 0x7FFF + ((u >> 16) & 1)) & 0xFFFFFFFF  # RNE to bf16
    return u >> 16


def test_element_definition_matches_python():
    got = synth.fill_bf16(6, 7, synth.T_W_DOWN, 0.02, offset=1000)
    want = [_element_python(7, synth.T_W_DOWN, 1000 + i, 0.02) for i in range(6)]
    assert list(got) == want
    gotf = synth.fill_f32(4, 3, synth.T_W_ROUTER, 0.02, offset=5)
    wantf = [_element_python(3, synth.T_W_ROUTER, 5 + i, 0.02, bf16=False) for i in range(4)]
    assert np.array_equal(gotf, np.array(wantf, dtype=np.float32))


def test_offsets_and_threads_consistent():
    full = synth.fill_bf16(100_003, 1, synth.T_X, 1.0)
    part = synth.fill_bf16(1000, 1, synth.T_X, 1.0, offset=50_000)
    assert np.array_equal(full[50_000:51_000], part)


def test_distribution():
    x = synth.fill_f32(1 << 20, 0, synth.T_X, 1.0)
    assert abs(x.mean()) < 5e-3
    assert abs(x.std() - 1.0) < 5e-3
    assert np.abs(x).max() <= 6.0
    # Irwin-Hall(12) kurtosis is 3 - 1.2/12 = 2.9
    kurt = float(((x - x.mean()) ** 4).mean() / x.var() ** 2)
    assert abs(kurt - 2.9) < 0.03


def test_gate_up_lazy_matches_full_and_zero_rows():
    cfg = synth.CONFIGS["tiny"].replace(zero_rows_pct=71)
    inp = synth.host_inputs(cfg, seed=2)
    full = inp.gate_up_all()
    for e in (0, 5, 15):
        assert np.array_equal(full[e], inp.gate_up(e))
    m = inp.zero_mask
    nz = (71 * cfg.I) // 100
    assert (m.sum(axis=1) == nz).all()
    for e in (0, 7):
        gate_zero = (full[e, :cfg.I] == 0).all(axis=1)
        up_zero = (full[e, cfg.I:] == 0).all(axis=1)
        assert np.array_equal(gate_zero, m[e].astype(bool))
        assert np.array_equal(up_zero, m[e].astype(bool))
    # down stays dense
    assert (inp.down_all() != 0).mean() > 0.99


def test_permutation_is_permutation():
    p = synth.permutation(512, 0, synth.T_ZIPF_PERM)
    assert sorted(p.tolist()) == list(range(512))
    assert not np.array_equal(p, np.arange(512))


def test_zipf_bias_formula():
    cfg = synth.CONFIGS["t24_skewed"]
    b = synth.zipf_bias(cfg, 0)
    p = synth.permutation(cfg.E, 0, synth.T_ZIPF_PERM)
    for e in (0, 1, 100, 511):
        assert b[e] == np.float32(-1.1 * math.log(1 + int(p[e])))
    assert b.max() == 0.0  # rank 1 expert
    assert np.isclose(b.min(), -1.1 * math.log(512), rtol=1e-6)
