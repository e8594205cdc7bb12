"""Error measures used by the parity tests (relative L1 and max-abs)."""
import numpy as np

# Bars for floating-point outputs against the float64 oracle: max-abs error and relative L1
# error (sum |gpu - ref| / sum |ref|).
MAX_ABS = 2e-2
MEAN_REL = 5e-3


def errors(gpu, ref):
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    d = np.abs(gpu - ref)
    return float(d.max()) if d.size else 0.0, float(d.sum() / max(np.abs(ref).sum(), 1e-300))


def row_scaled_max_abs(gpu, ref):
    """Max-abs error with each row divided by the oracle row's RMS (unit-scale hidden states)."""
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    rms = np.sqrt(np.mean(ref * ref, axis=-1, keepdims=True))
    return float(np.max(np.abs(gpu - ref) / np.maximum(rms, 1e-30)))


def check_readings(got, refs, what, row_scaled=True):
    """Assert the bars against each precision reading of the oracle in `refs` ({name: reference}).

    Hidden states are compared with the row-scaled max-abs (each row divided by the oracle row's RMS);
    logits with the raw max-abs. The raw max-abs and the relative L1 error are printed for every
    reading, so the test output records the numbers behind each verdict.
    """
    for name, ref in refs.items():
        raw, rel = errors(got, ref)
        mx = row_scaled_max_abs(got, ref) if row_scaled else raw
        print(f"{what} vs {name}: {'row-scaled ' if row_scaled else ''}max-abs {mx:.4g}, raw max-abs {raw:.4g}, "
              f"relative L1 {rel:.4g}")
        assert mx <= MAX_ABS and rel <= MEAN_REL, (what, name, mx, rel)
