"""The FP8 page dequantisation of the tensor-core decode, modelled on the CPU.

The kernel turns an e4m3 code into fp16 exactly, widens it to fp32 (exact), multiplies by the
token's fp32 scale (one rounding to fp32) and packs to bf16 (round to nearest even): the value
it feeds the tensor core is bf16(fp32(code * scale)).  The oracle uses code * scale exactly.
The model checks, for every finite code and scales over the whole range the append produces,
that this is within one bf16 ulp of the correctly rounded product, and within 2^-8 relative of
the exact value wherever that value is a normal number: the rounding a bf16 cache applies on
write.
"""
import numpy as np
import torch


def _decode_e4m3():
    codes = np.arange(256, dtype=np.uint8)
    v = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    ok = ~np.isnan(v)
    return codes[ok], v[ok]


def _bf16(x32):
    """fp32 -> bf16, round to nearest even (the kernel's pack)."""
    return torch.from_numpy(np.asarray(x32, dtype=np.float32)).to(torch.bfloat16).to(torch.float64).numpy()


def _bf16_rne(x64):
    """The correctly rounded bf16 of an fp64 value: 8 significant bits, nearest even (quantum
    2^-133 below 2^-126)."""
    x = np.asarray(x64, dtype=np.float64)
    _, e = np.frexp(x)
    q = np.where(np.abs(x) >= 2.0 ** -126, np.ldexp(1.0, e - 8), 2.0 ** -133)
    return np.rint(x / q) * q


def test_codes_are_exact_in_fp16_and_fp32():
    codes, v = _decode_e4m3()
    as16 = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float16).to(torch.float64).numpy()
    assert np.array_equal(as16, v)
    assert np.array_equal(v.astype(np.float32).astype(np.float64), v)


def test_kernel_dequantisation_is_one_bf16_rounding_of_the_exact_value():
    codes, v = _decode_e4m3()
    rng = np.random.default_rng(3)
    # per-token scales amax/448 over amax from tiny to large, plus the append's special values
    scales = np.concatenate([np.float32(np.exp(rng.uniform(np.log(1e-30), np.log(1e6), 3000))),
                             np.array([1.0, np.finfo(np.float32).tiny, 1.0 / 448, 0.0123], np.float32)])
    worst_rel = 0.0
    for sc in scales.astype(np.float32):
        exact = v * np.float64(sc)
        kernel = _bf16((v.astype(np.float32) * np.float32(sc)).astype(np.float32))
        want = _bf16_rne(exact)
        # one bf16 ulp at the correctly rounded value (2^-133 in the subnormal range)
        mag = np.maximum(np.abs(want), 2.0 ** -126)
        ulp = 2.0 ** (np.floor(np.log2(mag)) - 7)
        ulps = np.abs(kernel - want) / ulp
        assert ulps.max() <= 1.0
        normal = np.abs(exact) >= 2.0 ** -126  # relative bound where bf16 has its full precision
        if normal.any():
            rel = np.abs(kernel[normal] - exact[normal]) / np.abs(exact[normal])
            worst_rel = max(worst_rel, float(rel.max()))
        assert np.all(kernel[exact == 0] == 0)
    assert worst_rel <= 2.0 ** -8


def test_reference_rounding_matches_a_library_for_fp32_inputs():
    rng = np.random.default_rng(4)
    x = np.float32(rng.standard_normal(100000) * np.exp(rng.uniform(-80, 80, 100000)))
    assert np.array_equal(_bf16_rne(x.astype(np.float64)), _bf16(x))
