"""Helpers of the GPU parity tests: tolerances and comparisons against the oracle."""
import numpy as np
import torch

# GPU-vs-oracle bars, both with fp32 accumulation on the GPU:
#   fp32 inputs: max |err| <= 1e-5;  bf16 inputs: max |err| <= 2e-2 and mean |err| <= 2e-3.
TOL = {torch.float32: dict(max_abs=1e-5, mean_abs=1e-5),
       torch.bfloat16: dict(max_abs=2e-2, mean_abs=2e-3)}
LSE_TOL = {torch.float32: 1e-5, torch.bfloat16: 2e-3}


def to_np(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float32).numpy().astype(np.float64)


def assert_close(got: torch.Tensor, ref: np.ndarray, dtype, what=""):
    g = to_np(got)
    assert g.shape == ref.shape, (what, g.shape, ref.shape)
    assert np.all(np.isfinite(g)), f"{what}: non-finite output"
    err = np.abs(g - ref)
    tol = TOL[dtype]
    assert err.max() <= tol["max_abs"], f"{what}: max |err| {err.max():.3e} > {tol['max_abs']}"
    assert err.mean() <= tol["mean_abs"], f"{what}: mean |err| {err.mean():.3e} > {tol['mean_abs']}"
    return float(err.max()), float(err.mean())


def assert_lse_close(got: torch.Tensor, ref: np.ndarray, dtype, what=""):
    g = to_np(got)
    both_inf = np.isneginf(g) & np.isneginf(ref)
    with np.errstate(invalid="ignore"):   # -inf - -inf where both are -inf: masked below
        err = np.where(both_inf, 0.0, np.abs(g - ref))
    assert np.all(np.isfinite(err)), f"{what}: lse infinite where the oracle is finite"
    # lse is an fp32 statistic either way; a bf16 input only changes the scores' inputs
    assert err.max() <= LSE_TOL[dtype] * max(1.0, float(np.abs(ref[~both_inf]).max(initial=1.0))), \
        f"{what}: lse max |err| {err.max():.3e}"


def assert_close_stored(got: torch.Tensor, ref: np.ndarray, dtype, what=""):
    """For values the path stores in the input dtype that are not attention outputs (the
    projected and turned keys and values a fused block writes into its cache): unit-variance
    projections reach magnitudes of 5 and more over millions of rows, where one bf16 rounding
    step alone is up to 2^-9 |v| (0.016 at 5), so the max bar applies to |err| / max(1, |ref|);
    the mean bar is unchanged."""
    g = to_np(got)
    assert g.shape == ref.shape, (what, g.shape, ref.shape)
    assert np.all(np.isfinite(g)), f"{what}: non-finite output"
    err = np.abs(g - ref)
    rel = err / np.maximum(1.0, np.abs(ref))
    tol = TOL[dtype]
    assert rel.max() <= tol["max_abs"], f"{what}: max |err|/max(1,|ref|) {rel.max():.3e} > {tol['max_abs']}"
    assert err.mean() <= tol["mean_abs"], f"{what}: mean |err| {err.mean():.3e} > {tol['mean_abs']}"
