"""Shared helpers of the parity tests: error statistics and the tolerance of the layer.

Tolerance (stated for the layer's outputs, bf16 inputs with fp32 accumulation):
max |gpu - ref| <= 1e-2 * RMS(ref) and mean relative error
sum |gpu - ref| / sum |ref| <= 2e-3, against the fp64 oracle.
"""
import numpy as np

MAX_ABS_OVER_RMS = 1e-2
MEAN_REL = 2e-3
NEAR_TIE_GAP = 1e-5


def err_stats(gpu, ref):
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    d = np.abs(gpu - ref)
    rms = float(np.sqrt(np.mean(ref * ref)))
    return {"max_abs_over_rms": float(d.max() / rms) if d.size else 0.0,
            "mean_rel": float(d.sum() / np.abs(ref).sum()) if d.size else 0.0,
            "rms": rms}


def assert_layer_close(gpu, ref, what=""):
    s = err_stats(gpu, ref)
    assert np.isfinite(gpu).all(), f"{what}: non-finite output"
    assert s["max_abs_over_rms"] <= MAX_ABS_OVER_RMS, f"{what}: {s}"
    assert s["mean_rel"] <= MEAN_REL, f"{what}: {s}"
    return s


def id_sets_match(gpu_ids, ref_ids, ref_gap, ref_logits=None):
    """Exact set equality of routing ids per token, except near-ties.

    Returns the indices of near-tie tokens whose sets differ (gap < 1e-5 on the fp64
    logits). For those the GPU's set must still be valid: every chosen expert's fp64
    logit lies within 1e-5 of the k-th largest.
    """
    T, k = ref_ids.shape
    differ = []
    for t in range(T):
        a = set(int(v) for v in gpu_ids[t])
        b = set(int(v) for v in ref_ids[t])
        if a == b:
            continue
        assert ref_gap[t] < NEAR_TIE_GAP, f"token {t}: ids {sorted(a)} != {sorted(b)}, gap {ref_gap[t]}"
        assert len(a) == k
        if ref_logits is not None:
            kth = np.sort(ref_logits[t])[::-1][k - 1]
            assert all(ref_logits[t, e] >= kth - NEAR_TIE_GAP for e in a), f"token {t}: invalid near-tie set"
        differ.append(t)
    return differ
