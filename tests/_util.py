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


def assert_stored(gpu, ref, dtype: str, what: str, acc_tol: float = 2e-3):
    """An output stored in the input dtype (the chunk memories dH): every element within one storage
    rounding of the oracle's value (half an ulp, doubled for a sum that may sit on the other side of a
    rounding boundary: 2^-8 |ref| for bf16, 2^-23 |ref| for fp32) plus acc_tol * rms(ref) for the
    accumulation (fp16 products in the tensor-core path: ~5e-4 of rms). A max|err|/rms bound cannot hold
    for a bf16-stored tensor whose max/rms exceeds 10, as dH does with chunks of 32 tokens or fewer."""
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    ulp = 2.0 ** -8 if dtype == "bf16" else 2.0 ** -23
    rms = float(np.sqrt(np.mean(ref ** 2))) if ref.size else 0.0
    excess = np.abs(gpu - ref) - (ulp * np.abs(ref) + acc_tol * rms)
    worst = float(np.max(excess)) if excess.size else 0.0
    assert worst <= 0.0, f"{what}: an element exceeds one storage rounding + {acc_tol:g} rms by {worst:.3e} (rms {rms:.3e})"
    return worst


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
