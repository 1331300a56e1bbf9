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


# Weight gradients are fp32 sums over an expert's n rows of exact bf16 x bf16 products. A
# sum of n terms with fp32 additions (rounded or truncated, in any order and grouping) is
# within (n - 1) * 2^-23 * sum|terms| of the exact sum to first order; the bar takes twice
# that, plus one final rounding (two when the result is added into a prior fp32 value).
def assert_close_fp32_sums(got, ref, abs_sum, n_terms: int, what: str = "", added=False):
    g = np.asarray(got, np.float64)
    r = np.asarray(ref, np.float64)
    assert g.shape == r.shape, (what, g.shape, r.shape)
    assert np.all(np.isfinite(g)), f"{what}: non-finite values"
    u = 2.0 ** -23
    bound = 2.0 * n_terms * u * np.asarray(abs_sum, np.float64) + (2 if added else 1) * u * np.abs(r)
    err = np.abs(g - r)
    bad = err > bound + 1e-38
    assert not bad.any(), (f"{what}: {int(bad.sum())} elements beyond the fp32 summation bound "
                           f"(worst excess {float((err - bound).max()):.3e})")
    nr = np.linalg.norm(r)
    return {"rel_fro": float(np.linalg.norm(g - r) / max(nr, 1e-30)),
            "max_err_over_bound": float((err / np.maximum(bound, 1e-38)).max()) if err.size else 0.0}


# ----------------------------------------------------------------------------- guard bands
#
# An out-of-bounds check for the GPU tests in place of a memory sanitizer: every output buffer
# is carved out of a larger allocation with GUARD_BYTES of a sentinel byte before and after
# it. A kernel that stores past either end of its buffer (a ragged tail, a wrong row) changes
# a guard byte, and the check after the test finds it.

GUARD_BYTES = 64 << 10
GUARD_SENTINEL = 0xA5


class GuardedAllocator:
    def __init__(self):
        self.regions = []

    def reset(self):
        self.regions = []

    def __call__(self, shape, dtype, device=None, fill_byte=0xFF):
        """A tensor of `shape` and `dtype` inside guard bands; its own bytes are `fill_byte`
        (0xFF: NaN for floating types, -1 for integers) so that unwritten outputs show."""
        device = device if device is not None else torch.device("cuda:0")
        shape = tuple(int(d) for d in shape)
        n = int(np.prod(shape)) * torch.empty((), dtype=dtype).element_size()
        tail = GUARD_BYTES + ((-n) % 256)
        raw = torch.empty(GUARD_BYTES + n + tail, dtype=torch.uint8, device=device)
        raw[:GUARD_BYTES].fill_(GUARD_SENTINEL)
        raw[GUARD_BYTES + n:].fill_(GUARD_SENTINEL)
        inner = raw[GUARD_BYTES:GUARD_BYTES + n]
        inner.fill_(fill_byte)
        self.regions.append((raw, n))
        return inner.view(dtype).view(shape)

    def full(self, shape, value, dtype, device=None):
        t = self(shape, dtype, device)
        t.fill_(value)
        return t

    def zeros(self, shape, dtype, device=None):
        return self(shape, dtype, device, fill_byte=0)

    def for_device(self, device):
        """The allocator as LayerBuffers / LayerGrads / MxBuffers.allocate take it."""
        return lambda shape, dtype: self(shape, dtype, device)

    def check(self):
        """Every guard byte still holds the sentinel (synchronises first)."""
        if not self.regions:
            return
        torch.cuda.synchronize()
        bad = []
        for i, (raw, n) in enumerate(self.regions):
            head = raw[:GUARD_BYTES]
            tail = raw[GUARD_BYTES + n:]
            nh = int((head != GUARD_SENTINEL).sum().item())
            nt = int((tail != GUARD_SENTINEL).sum().item())
            if nh or nt:
                bad.append(f"buffer {i} ({n} bytes): {nh} guard bytes changed before it, "
                           f"{nt} after it")
        assert not bad, "out-of-bounds writes: " + "; ".join(bad)


GUARD = GuardedAllocator()
