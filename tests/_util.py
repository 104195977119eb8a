"""Helpers shared by the GPU parity tests: upload seeded inputs, compare with tolerances.

Tolerances (from the float arithmetic): max |gpu - ref| <= tol * rms(ref) with
tol = 1e-4 for fp32 storage and 2e-2 for bf16 storage (fp32 accumulation);
lse is compared on finite entries and its -inf mask must match exactly.
"""
import numpy as np

TOL = {"f32": 1e-4, "bf16": 2e-2}


def to_dev(x, device="cuda"):
    """Upload a workloads.Stored (or an fp32 numpy array) to the GPU, keeping its exact bits."""
    import torch

    if hasattr(x, "storage") and hasattr(x, "dtype") and x.dtype in ("bf16", "f32"):
        if x.dtype == "bf16":
            t = torch.from_numpy(np.ascontiguousarray(x.storage).view(np.int16)).view(torch.bfloat16)
        else:
            t = torch.from_numpy(np.ascontiguousarray(x.storage))
        return t.to(device)
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(device)


def to_f64(t) -> np.ndarray:
    return t.detach().double().cpu().numpy()


def rel_err(gpu, ref) -> float:
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    rms = float(np.sqrt(np.mean(ref ** 2)))
    if rms == 0.0:
        return float(np.max(np.abs(gpu - ref))) if gpu.size else 0.0
    return float(np.max(np.abs(gpu - ref))) / rms


def assert_close(gpu, ref, dtype: str, what: str):
    e = rel_err(gpu, ref)
    assert e <= TOL[dtype], f"{what}: max|err|/rms = {e:.3e} > {TOL[dtype]:.0e}"
    return e


def assert_lse(gpu, ref, dtype: str, what: str = "lse"):
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    np.testing.assert_array_equal(np.isneginf(gpu), np.isneginf(ref), err_msg=f"{what}: -inf mask differs")
    fin = np.isfinite(ref)
    assert np.all(np.isfinite(gpu[fin])), f"{what}: non-finite where the oracle is finite"
    if fin.any():
        return assert_close(gpu[fin], ref[fin], dtype, what)
    return 0.0


def layer_inputs_dev(inp):
    return {k: to_dev(inp[k]) for k in ("X", "B", "C", "Q", "E")} | {
        "logA": to_dev(inp["logA"]), "g": to_dev(inp["g"])}
