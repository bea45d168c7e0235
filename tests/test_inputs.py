"""Pins for the seeded input generator that both sides of every parity check draw from:
the counter-based SplitMix64 against its published sequence, the distributions it
produces, the bf16 rounding against PyTorch's, and the workload recipes."""
import math

import numpy as np
import pytest

from long_context_attention_fwd_b200 import inputs as I

M64 = (1 << 64) - 1


def _splitmix64_sequential(state: int, n: int):
    """SplitMix64 as published, in its sequential form: advance the state by the golden
    gamma, then apply the finaliser."""
    out = []
    for _ in range(n):
        state = (state + 0x9E3779B97F4A7C15) & M64
        z = state
        z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & M64
        z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & M64
        out.append(z ^ (z >> 31))
    return out


def test_splitmix64_known_answers():
    # the first outputs of SplitMix64 seeded with 0, as published with the generator
    want = [0xE220A8397B1DCDAF, 0x6E789E6AA1B965F4, 0x06C45D188009454F, 0xF88BB8A8724C81EC]
    assert [int(x) for x in I.raw_u64(0, 0, 4)] == want


@pytest.mark.parametrize("key,start", [(0x0123456789ABCDEF, 0), (I.stream_key(7, I.TAG_V), 1000)])
def test_counter_form_equals_sequential_form(key, start):
    seq = _splitmix64_sequential((key + start * 0x9E3779B97F4A7C15) & M64, 64)
    assert [int(x) for x in I.raw_u64(key, start, 64)] == seq


def test_uniform_range_and_moments():
    u = I.uniform(I.stream_key(1, 1), 1 << 20)
    assert u.min() >= 0.0 and u.max() < 1.0
    n = u.size
    assert abs(u.mean() - 0.5) < 5 * math.sqrt(1 / 12 / n)
    assert abs(u.var() - 1 / 12) < 0.002


def test_normal_moments_and_chunking():
    key = I.stream_key(2, I.TAG_Q)
    n = 3 * (1 << 22) + 5          # several chunks filled in parallel, odd count
    x = I.normal(key, n)
    assert np.isfinite(x).all()
    assert abs(x.mean()) < 5 / math.sqrt(n)
    assert abs(x.var() - 1.0) < 5 * math.sqrt(2 / n)
    kurt = np.mean(x ** 4) / x.var() ** 2
    assert abs(kurt - 3.0) < 0.02
    # a prefix is the same whichever count it was drawn with (counter-based stream)
    assert np.array_equal(I.normal(key, 1001), x[:1001])


def test_bf16_rounding_matches_torch():
    torch = pytest.importorskip("torch")
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(100000) * 10.0 ** rng.integers(-8, 8, 100000),
                        # exact ties between two bf16 values: both even and odd lower neighbours
                        np.array([1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, -1.0 - 2.0 ** -8,
                                  0.0, -0.0, 1e-40, 3.0e38])])
    ours = I.to_bf16_bits(x)
    theirs = torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16).view(torch.int16).numpy()
    assert np.array_equal(ours, theirs.view(np.uint16))
    back = I.bf16_bits_to_f64(ours)
    assert np.array_equal(I.to_bf16_bits(back), ours)   # exact round trip


def test_outlier_fraction():
    key, okey = I.stream_key(3, I.TAG_Q), I.stream_key(3, I.TAG_OUT_Q)
    n = 1 << 20
    plain = I.bf16_bits_to_f64(I.normal_bf16(key, (n,)))
    spiked = I.bf16_bits_to_f64(I.normal_bf16(key, (n,), outlier_key=okey, outlier_p=0.01,
                                              outlier_mult=8.0))
    changed = plain != spiked
    frac = changed.mean()
    assert abs(frac - 0.01) < 5 * math.sqrt(0.01 * 0.99 / n)
    np.testing.assert_allclose(spiked[changed], plain[changed] * 8.0, rtol=2 ** -7)


def test_varlen_recipe():
    lens = I.varlen_lengths(99, 32768, 512, 8192)
    assert sum(lens) == 32768
    assert all(512 <= L <= 8192 for L in lens[:-1]) and 1 <= lens[-1] <= 8192
    assert lens == I.varlen_lengths(99, 32768, 512, 8192)
    cu = I.cu_seqlens_from(lens)
    assert cu[0] == 0 and cu[-1] == 32768 and np.all(np.diff(cu) == np.array(lens))
    # the packed workload's lengths are the recipe's draw for its seed
    w = I.workload(3)
    assert w.varlen == I.varlen_lengths(20261202 + 3, 32768, 512, 8192)


def test_streams_are_distinct_and_reproducible():
    a = I.normal(I.stream_key(5, I.TAG_Q), 1000)
    b = I.normal(I.stream_key(5, I.TAG_K), 1000)
    c = I.normal(I.stream_key(6, I.TAG_Q), 1000)
    assert np.array_equal(a, I.normal(I.stream_key(5, I.TAG_Q), 1000))
    assert abs(np.corrcoef(a, b)[0, 1]) < 0.15 and abs(np.corrcoef(a, c)[0, 1]) < 0.15
    assert len({I.stream_key(s, t) for s in range(4) for t in range(1, 9)}) == 32
