"""Helpers shared by the GPU tests: the acceptance bound and small runners."""
import numpy as np

COS_MIN = 0.999      # per-token cosine similarity
REL_MAX = 2e-2       # max |err| per row relative to the reference row's RMS


def row_metrics(got, ref):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    num = (got * ref).sum(1)
    den = np.linalg.norm(got, axis=1) * np.linalg.norm(ref, axis=1)
    cos = np.where(den > 0, num / np.maximum(den, 1e-300), 1.0)
    rms = np.sqrt((ref ** 2).mean(1))
    err = np.abs(got - ref).max(1)
    return cos, err / np.maximum(rms, 1e-300)


def assert_rows_close(got, ref, what="", cos_min=COS_MIN, rel_max=REL_MAX):
    """Per-token cosine >= cos_min and max |err| <= rel_max * row RMS."""
    cos, rel = row_metrics(got, ref)
    worst_c, worst_r = int(np.argmin(cos)), int(np.argmax(rel))
    print(f"[parity] {what}: rows {len(cos)} min cos {cos.min():.7f} max rel err {rel.max():.4g}")
    assert cos.min() >= cos_min and rel.max() <= rel_max, (
        f"{what}: min cos {cos.min():.6f} (row {worst_c}), max rel err {rel.max():.4g} "
        f"(row {worst_r}) over {len(cos)} rows")
    return cos.min(), rel.max()


def assert_bf16_output_close(got, ref, what="", atol=None, rel=2.0 ** -8, kind="bf16"):
    """Bound for a kernel whose output is stored in bf16 from fp32 arithmetic:
    round-to-nearest-even to 8 significant bits errs by at most 2^-8 |v| (rel),
    plus a small absolute term for the fp32 arithmetic (default 1e-3 of the row
    RMS)."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    if atol is None:
        atol = 1e-3 * np.sqrt((ref ** 2).mean(1, keepdims=True))
    excess = np.abs(got - ref) - (rel * np.abs(ref) + atol)
    i = np.unravel_index(int(np.argmax(excess)), excess.shape)
    assert excess.max() <= 0, (f"{what}: element {i} got {got[i]:.6g} ref {ref[i]:.6g} "
                               f"exceeds the {kind} bound by {excess[i]:.3g}")


def assert_f16_output_close(got, ref, what="", atol=None):
    """The same for an fp16 output: 11 significant bits, at most 2^-11 |v|."""
    assert_bf16_output_close(got, ref, what, atol, rel=2.0 ** -11, kind="fp16")
