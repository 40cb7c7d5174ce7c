"""Comparison helpers and tolerances shared by the parity tests.

Tolerances (stated with the workloads): float32 inputs, relative L2 error
<= 1e-5; bfloat16 inputs with float32 accumulation, relative L2 <= 1e-2 and
max |error| <= 3e-2 * RMS(reference).  Every comparison is made over the
whole tensor and per head, so that a head with a small decay cannot hide
behind the others.
"""

import numpy as np

F32_REL_L2 = 1e-5
BF16_REL_L2 = 1e-2
BF16_MAX_ABS_OVER_RMS = 3e-2
# Unit roundoff of bfloat16 (8 significant bits).  When an output is STORED as
# bfloat16, the store alone moves each element by up to BF16_U * |value|; for
# heavy-tailed outputs (gated values reach ~40x their RMS) that exceeds the
# max-abs bound above, which is about accumulated arithmetic error.  So for a
# bf16-stored output the elementwise bound is 3e-2 * RMS(ref) + BF16_U * |ref|;
# the arithmetic itself is checked against the plain bound with float32
# outputs of the same kernels.
BF16_U = 2.0 ** -8


def rel_l2(got, ref):
    got, ref = np.asarray(got, np.float64), np.asarray(ref, np.float64)
    den = np.linalg.norm(ref)
    return float(np.linalg.norm(got - ref) / den) if den > 0 else float(np.linalg.norm(got))


def max_abs_over_rms(got, ref):
    got, ref = np.asarray(got, np.float64), np.asarray(ref, np.float64)
    rms = np.sqrt(np.mean(ref ** 2))
    err = np.max(np.abs(got - ref)) if got.size else 0.0
    return float(err / rms) if rms > 0 else float(err)


def assert_close(got, ref, kind, head_axis=None, what="", stored_bf16=False):
    """kind: 'f32' or 'bf16' (tolerance class of the computation).  head_axis:
    axis of the heads for per-head checks.  stored_bf16: the output was stored
    as bfloat16 (adds the store's rounding to the max-abs bound)."""
    got, ref = np.asarray(got, np.float64), np.asarray(ref, np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    groups = [(None, got, ref)]
    if head_axis is not None:
        for h in range(got.shape[head_axis]):
            groups.append((h, np.take(got, h, axis=head_axis), np.take(ref, h, axis=head_axis)))
    for h, g, r in groups:
        e = rel_l2(g, r)
        tag = f"{what} head={h}" if h is not None else what
        if kind == "f32":
            assert e <= F32_REL_L2, f"{tag}: rel-L2 {e:.3e} > {F32_REL_L2}"
        else:
            assert e <= BF16_REL_L2, f"{tag}: rel-L2 {e:.3e} > {BF16_REL_L2}"
            if stored_bf16:
                rms = np.sqrt(np.mean(r ** 2))
                excess = np.abs(g - r) - (BF16_MAX_ABS_OVER_RMS * rms + BF16_U * np.abs(r))
                assert excess.max(initial=-1.0) <= 0.0, (
                    f"{tag}: |err| exceeds 3e-2*RMS + u*|ref| by {excess.max():.3e}")
            else:
                m = max_abs_over_rms(g, r)
                assert m <= BF16_MAX_ABS_OVER_RMS, f"{tag}: max-abs/RMS {m:.3e} > {BF16_MAX_ABS_OVER_RMS}"
