"""Shared test helpers: tensor <-> bit conversions and the floating-point acceptance bar."""
import numpy as np
import torch

# Acceptance bar for bf16 outputs (fp32 accumulate) against the fp64 oracle:
# relative Frobenius error <= 5e-3 and max |err| <= 3e-2 * rms(reference).
REL_FRO_TOL = 5e-3
MAX_ABS_RMS_TOL = 3e-2
# bf16 spacing exceeds 3e-2 * rms for elements above ~7.7 * rms, so a correctly computed
# value that lies next to a rounding tie may round to the neighbouring bf16 value (fp32 vs
# fp64 accumulation). Such an element passes only if it is exactly one bf16 step from the
# oracle, and there may be at most this fraction of them.
MAX_ONE_ULP_FLIP_FRACTION = 1e-4


def bits(t: torch.Tensor) -> np.ndarray:
    """bf16 tensor (any device) -> numpy uint16 bit patterns."""
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


def f64(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def bf16_ulp(b: np.ndarray) -> np.ndarray:
    """Spacing of bf16 values at each bf16 bit pattern (2^-133 in the subnormal range)."""
    e = (np.asarray(b, dtype=np.int64) >> 7) & 0xFF
    return np.ldexp(1.0, np.maximum(e, 1) - 134)


def assert_close_bf16(got_bits: np.ndarray, ref_bits: np.ndarray, what: str = "", inherited=None):
    """The bar above. `inherited` (end-to-end checks only): per-element bound on the
    difference carried in from one-step flips of the bf16 inputs of the last stage; an
    element beyond the max-abs bar is then accepted if it lies within that bound plus one
    step of its own rounding."""
    g, r = f64(got_bits), f64(ref_bits)
    assert g.shape == r.shape, (what, g.shape, r.shape)
    assert np.all(np.isfinite(g)), f"{what}: non-finite values"
    diff = g - r
    nr = np.linalg.norm(r)
    rel = np.linalg.norm(diff) / max(nr, 1e-30)
    rms = nr / np.sqrt(max(r.size, 1))
    assert rel <= REL_FRO_TOL, f"{what}: relative Frobenius error {rel:.3e} > {REL_FRO_TOL}"
    over = np.abs(diff) > MAX_ABS_RMS_TOL * rms
    n_over = int(over.sum())
    if n_over:
        gb = np.asarray(got_bits, np.int32)[over]
        rb = np.asarray(ref_bits, np.int32)[over]
        same_sign = (gb >> 15) == (rb >> 15)
        one_step = same_sign & (np.abs(gb - rb) == 1)
        if inherited is not None:
            bound = np.asarray(inherited, np.float64)[over] + bf16_ulp(rb)
            one_step |= np.abs(diff[over]) <= bound
        worst = np.abs(diff).max() / rms
        assert one_step.all(), (
            f"{what}: {int((~one_step).sum())} elements off by more than one bf16 step (plus any "
            f"inherited flips) and more "
            f"than {MAX_ABS_RMS_TOL} * rms (worst {worst:.3e} * rms)")
        limit = MAX_ONE_ULP_FLIP_FRACTION * r.size + 2
        assert n_over <= limit, (
            f"{what}: {n_over} one-step rounding flips above {MAX_ABS_RMS_TOL} * rms "
            f"(limit {limit:.0f} of {r.size})")
    mx = float(np.abs(diff).max()) / max(rms, 1e-30) if diff.size else 0.0
    return {"rel_fro": float(rel), "max_abs_over_rms": mx, "one_step_flips_over_bar": n_over,
            "exact_fraction": float((diff == 0).mean()) if diff.size else 1.0}
