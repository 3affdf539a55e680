"""The number-format facts the FP8 path is built on, checked on the CPU over all 256 E4M3
codes (values from the oracle's decoder, which the pins fix):

* every finite E4M3 value is exactly an f16 value (the decode/verify tasks convert codes to
  f16 and multiply in f16) and exactly a bf16 value (the tensor-core tasks read bf16 copies
  of the codes), so neither conversion rounds;
* a product of a code value and an f16 / bf16 query element is exact in fp32 (the MMAs
  accumulate in fp32), so the only rounding before the accumulation is the input's own.
"""
import numpy as np
import torch

import oracle


def finite_code_values():
    v = oracle.e4m3_decode(np.arange(256))
    return v[np.isfinite(v)]


def test_every_e4m3_value_is_exact_in_f16_and_bf16():
    v = finite_code_values()
    assert len(v) == 254                       # 256 codes minus the two NaN codes
    t = torch.from_numpy(v)
    for dt in (torch.float16, torch.bfloat16):
        back = t.to(dt).to(torch.float64).numpy()
        assert np.array_equal(back, v), dt
    # and the largest / smallest magnitudes sit well inside both formats' normal ranges
    # (f16's smallest normal is 2^-14; E4M3's smallest subnormal is 2^-9)
    mags = np.abs(v[v != 0])
    assert mags.min() == 2.0 ** -9 and mags.max() == 448.0


def test_code_times_input_is_exact_in_fp32():
    v = finite_code_values()
    # E4M3 values carry at most 4 significant bits, bf16 at most 8 and f16 at most 11: a
    # product has at most 15 significant bits, inside fp32's 24
    rng = np.random.default_rng(7)
    q = torch.randn(4096, generator=torch.Generator().manual_seed(7))
    for dt in (torch.bfloat16, torch.float16):
        qv = q.to(dt).to(torch.float64).numpy()
        a = rng.choice(v, size=qv.size)
        exact = a * qv                                          # float64: exact for these
        f32 = (torch.from_numpy(a).float() * torch.from_numpy(qv).float()).double().numpy()
        assert np.array_equal(f32, exact), dt
