"""The bit-level rules the many-row attention kernel relies on, checked on
the CPU against torch's own conversions.

* fp8 (e4m3fn) codes are widened to bf16 through the hardware e4m3x2 -> f16x2
  conversion followed by moving the f16 fields into bf16 position: magnitude
  >> 3, exponent rebias by 112 << 7 for nonzero halves, sign kept.  Every
  e4m3 value is a normal f16 or zero with at most 3 mantissa bits, so the
  result must equal torch's e4m3 -> bf16 conversion exactly, for every pair
  of codes (NaN codes excepted: they only occur in unfilled token slots,
  which are masked or zeroed).
* The weights enter the bf16 products as hi = p with its low 16 bits
  cleared and lo = the fp32 remainder truncated the same way; hi + lo must
  be within 2^-14 of p (relative).
"""
import numpy as np
import torch


def _e4m3_to_f16_bits():
    codes = torch.arange(256, dtype=torch.uint8)
    f = codes.view(torch.float8_e4m3fn).to(torch.float32)
    h16 = f.to(torch.float16).view(torch.int16).numpy().astype(np.uint32) & 0xFFFF
    bf = f.to(torch.bfloat16).view(torch.int16).numpy().astype(np.uint32) & 0xFFFF
    return f.numpy(), h16, bf


def _widen_pair(h2):
    """The kernel's f16x2 -> bf16x2 field move, on uint32 arrays."""
    mag = (h2 >> 3) & 0x0FFF0FFF
    nz = ((mag + 0x0D000D00) & 0x10001000) >> 12
    return ((nz * 0x3800 + mag) | (h2 & 0x80008000)) & 0xFFFFFFFF


def test_e4m3_pairs_widen_to_bf16_exactly():
    f, h16, bf = _e4m3_to_f16_bits()
    lo, hi = np.meshgrid(np.arange(256), np.arange(256), indexing="ij")
    lo, hi = lo.ravel(), hi.ravel()
    finite = ~(np.isnan(f[lo]) | np.isnan(f[hi]))
    h2 = h16[lo] | (h16[hi] << 16)
    got = _widen_pair(h2.astype(np.uint64)).astype(np.uint64)
    want = (bf[lo] | (bf[hi] << 16)).astype(np.uint64)
    assert finite.sum() == 254 * 254
    assert np.array_equal(got[finite], want[finite])


def test_zero_codes_widen_to_signed_zero():
    f, h16, _ = _e4m3_to_f16_bits()
    for code, want in ((0x00, 0x0000), (0x80, 0x8000)):
        assert _widen_pair(np.array([h16[code]], dtype=np.uint64))[0] == want


def test_truncated_hi_lo_split_bound():
    rng = np.random.default_rng(0)
    # weights as the kernel forms them: 2^x for x up to the slack, times a scale
    p = (np.exp2(rng.uniform(-40.0, 16.0, 200_000)) * rng.uniform(0.001, 1.0, 200_000)).astype(np.float32)
    b = p.view(np.uint32)
    hi = (b & 0xFFFF0000).view(np.float32)
    r = (p - hi).astype(np.float32)                       # exact in fp32
    lo = (r.view(np.uint32) & 0xFFFF0000).view(np.float32)
    err = np.abs(p.astype(np.float64) - hi.astype(np.float64) - lo.astype(np.float64)) / p.astype(np.float64)
    assert np.all(r.astype(np.float64) == p.astype(np.float64) - hi.astype(np.float64))
    assert err.max() <= 2.0 ** -14
