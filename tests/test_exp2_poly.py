"""Error bound of the FMA-pipe exp2 used for part of the softmax probabilities.

The attention kernel evaluates 2^x for some elements as: clamp x >= -125, n = rint(x)
via the 1.5*2^23 rounding trick, f = x - n in [-0.5, 0.5], a cubic in f, and 2^n added
to the exponent field.  This test performs the same float32 operation sequence in numpy
and checks it against 2^x in float64 over the range the kernel feeds it (x <= 8):
relative error below 1e-4, far inside the bf16 rounding (2^-9) applied to P afterwards.
The device code itself is covered by the GPU parity tests."""
import numpy as np

C = [np.float32(v) for v in (0.999928057, 0.693260968, 0.242611140, 0.0551716685)]


def exp2_poly_f32(x):
    x = np.maximum(x.astype(np.float32), np.float32(-125.0))
    t = (x + np.float32(12582912.0)).astype(np.float32)
    n = (t - np.float32(12582912.0)).astype(np.float32)
    f = (x - n).astype(np.float32)
    q = (C[3] * f + C[2]).astype(np.float32)
    q = (q * f + C[1]).astype(np.float32)
    q = (q * f + C[0]).astype(np.float32)
    bits = q.view(np.uint32) + (t.view(np.uint32) << np.uint32(23))
    return bits.astype(np.uint32).view(np.float32)


def test_relative_error_bound():
    x = np.concatenate([np.linspace(-124.0, 8.0, 2_000_001, dtype=np.float32),
                        np.float32(np.arange(-124, 9)) + np.float32(0.5),
                        np.float32(np.arange(-124, 9))])
    got = exp2_poly_f32(x).astype(np.float64)
    want = np.exp2(x.astype(np.float64))
    rel = np.abs(got / want - 1.0)
    assert rel.max() < 1e-4, rel.max()


def test_large_negative_inputs_are_tiny():
    x = np.array([-126.0, -200.0, -1e30, -np.inf], dtype=np.float32)
    got = exp2_poly_f32(x)
    assert np.all(got >= 0) and np.all(got < 1e-37)
