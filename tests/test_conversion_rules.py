"""The bit-level rules the many-row attention kernel relies on, checked on
the CPU against torch's own conversions.

* The weights enter the bf16 products as hi = p with its low 16 bits
  cleared and lo = the fp32 remainder truncated the same way; hi + lo must
  be within 2^-14 of p (relative).
* fp8 caches: V is widened e4m3 -> f16 exactly for the f16 PV product, and
  each bf16 query row, scaled by a power of two, is split into two e4m3
  terms for the fp8 QK product, exactly for every element within 2^9 of the
  row's largest.
"""
import numpy as np
import torch


def _e4m3_to_f16_bits():
    codes = torch.arange(256, dtype=torch.uint8)
    f = codes.view(torch.float8_e4m3fn).to(torch.float32)
    h16 = f.to(torch.float16).view(torch.int16).numpy().astype(np.uint32) & 0xFFFF
    return f.numpy(), h16


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


def test_e4m3_widens_to_f16_exactly():
    """fp8 caches: V enters the PV product as f16 through the hardware
    e4m3x2 -> f16x2 conversion alone; every finite e4m3 value is an f16
    value, so the widening is exact (torch's conversion as the reference)."""
    f, h16 = _e4m3_to_f16_bits()
    finite = ~np.isnan(f)
    back = torch.from_numpy(h16.astype(np.int16)).view(torch.float16).to(torch.float64).numpy()
    assert np.array_equal(back[finite], f[finite].astype(np.float64))


def _q_split(q32):
    """The kernel's query split for the fp8 QK product, on float32 rows
    [n, 128]: each row scaled by 2^e with e = 7 - floor(log2 max|q|) (its
    largest element lands in [2^7, 2^8)), then q' = q1 + q2 with q1 =
    e4m3(q') and q2 = e4m3(q' - q1), both rounded to nearest even."""
    mx = np.abs(q32).max(axis=1, keepdims=True)
    e = np.where(mx > 0, 7 - np.floor(np.log2(np.where(mx > 0, mx, 1.0))), 0.0)
    qs = (q32 * np.exp2(e)).astype(np.float32)
    t = torch.from_numpy(qs)
    q1 = t.to(torch.float8_e4m3fn).to(torch.float32)
    q2 = (t - q1).to(torch.float8_e4m3fn).to(torch.float32)
    return qs, q1.numpy(), q2.numpy(), mx * np.exp2(e)


def test_two_term_e4m3_query_split_is_exact():
    """bf16 query rows (8 significant bits) split into two e4m3 terms (4
    each): exact for every element within 2^9 of the row's largest; below
    that the error stays under 2^-17 of the row's largest."""
    rng = np.random.default_rng(1)
    q = rng.standard_normal((4096, 128)) * np.exp2(rng.integers(-20, 20, (4096, 1)))
    q = torch.from_numpy(q.astype(np.float32)).to(torch.bfloat16).to(torch.float32).numpy()
    qs, q1, q2, rowmax = _q_split(q)
    assert np.all((rowmax >= 128) & (rowmax < 256))
    exact = np.abs(qs) >= rowmax * 2.0 ** -9
    assert np.array_equal((q1 + q2)[exact], qs[exact])
    err = np.abs(q1.astype(np.float64) + q2 - qs) / rowmax
    assert err.max() <= 2.0 ** -17
