"""Comparison rules between the CUDA path and the float64 oracle.

Attention outputs (16-bit KV, fp32 accumulation): elementwise
|gpu - ref| <= 2e-3 + ulp(out dtype, ref)  -- the absolute bound plus one
unit in the last place of the output format, since a correctly computed
result must still be rounded to fp16 / bf16 -- and a relative L2 error
<= 5e-3, so that tiny outputs at long contexts cannot pass vacuously.
FP8 KV: max-abs <= 3e-2 and relative L2 <= 1e-2 against the oracle run on
the dequantised FP8 values.  Byte and index results: bit-exact.

Prefill outputs are held to the same 16-bit rule: each chunk row is the
token-form attention of a query at its position, exactly what a decode
query computes.
"""
from __future__ import annotations

import numpy as np

ABS_TOL = {"f16": 2e-3, "bf16": 2e-3, "e4m3": 3e-2}
REL_L2_TOL = {"f16": 5e-3, "bf16": 5e-3, "e4m3": 1e-2}
MANT_BITS = {"f16": 10, "bf16": 7}
MIN_EXP = {"f16": -14, "bf16": -126}


def ulp(dtype: str, ref: np.ndarray) -> np.ndarray:
    """Spacing of the output format's numbers at |ref| (normal range; subnormal spacing below)."""
    a = np.abs(ref)
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    e = np.maximum(e, MIN_EXP[dtype])
    return np.exp2(e - MANT_BITS[dtype])


def to_f64(bits: np.ndarray, dtype: str) -> np.ndarray:
    if dtype == "f16":
        return bits.view(np.float16).astype(np.float64)
    import torch
    return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).double().numpy()


def attention_errors(out: np.ndarray, ref: np.ndarray) -> dict:
    err = np.abs(out - ref)
    denom = float(np.linalg.norm(ref.ravel()))
    return {"max_abs": float(err.max()) if err.size else 0.0,
            "rel_l2": float(np.linalg.norm((out - ref).ravel()) / denom) if denom > 0 else float(err.max() if err.size else 0.0)}


def attention_close(out: np.ndarray, ref: np.ndarray, kv_dtype: str, out_dtype: str):
    """(ok, report) for an attention output already converted to float64."""
    if out.shape != ref.shape:
        return False, {"shape": (out.shape, ref.shape)}
    if not np.all(np.isfinite(out)):
        return False, {"nonfinite": int((~np.isfinite(out)).sum())}
    rep = attention_errors(out, ref)
    if kv_dtype == "e4m3":
        ok = rep["max_abs"] <= ABS_TOL["e4m3"] and rep["rel_l2"] <= REL_L2_TOL["e4m3"]
    else:
        bound = ABS_TOL[kv_dtype] + ulp(out_dtype, ref)
        worst = float(np.max(np.abs(out - ref) - bound)) if out.size else -1.0
        rep["worst_excess"] = worst
        ok = worst <= 0.0 and rep["rel_l2"] <= REL_L2_TOL[kv_dtype]
    return ok, rep


def prefill_close(out: np.ndarray, ref: np.ndarray, dtype: str):
    """(ok, report) for a 16-bit prefill output in float64: the decode rule, unchanged (every chunk
    row is the same token-form attention as a decode query at its position)."""
    return attention_close(out, ref, dtype, dtype)
