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
    assert cos.min() >= cos_min and rel.max() <= rel_max, (
        f"{what}: min cos {cos.min():.6f} (row {worst_c}), max rel err {rel.max():.4g} "
        f"(row {worst_r}) over {len(cos)} rows")
    return cos.min(), rel.max()
