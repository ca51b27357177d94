"""Upload a generated Case to torch tensors on a device (layout only, no arithmetic)."""
from __future__ import annotations

import numpy as np
import torch

from .inputs import Case

_TORCH = {"bf16": torch.bfloat16, "fp16": torch.float16, "fp32": torch.float32}


def tensor(a: np.ndarray, dtype, device) -> torch.Tensor:
    """Exact conversion: `a` already holds values representable in `dtype`."""
    t = torch.from_numpy(np.ascontiguousarray(a))
    return t.to(device=device, dtype=dtype)


def case_tensors(case: Case, device) -> dict:
    """Device tensors of a Case; layer dicts use the field names of the binding's LayerWeights."""
    cfg = case.cfg
    dt = _TORCH[cfg.dtype]
    out = {
        "offsets": tensor(case.offsets, torch.int64, device),
        "timestamps": tensor(case.timestamps, torch.int64, device),
        "x": tensor(case.x, dt, device),
        "layers": [],
    }
    for lw in case.layers:
        out["layers"].append({
            "w1": tensor(lw.w1, dt, device),
            "b1": tensor(lw.b1, torch.float32, device),
            "w2": tensor(lw.w2, dt, device),
            "b2": tensor(lw.b2, torch.float32, device),
            "rab_pos": tensor(lw.rab_pos, torch.float32, device),
            "rab_time": tensor(lw.rab_time, torch.float32, device),
            "ln_gamma": None if lw.ln_gamma is None else tensor(lw.ln_gamma, torch.float32, device),
            "ln_beta": None if lw.ln_beta is None else tensor(lw.ln_beta, torch.float32, device),
        })
    if case.cand_emb is not None:
        out["cand_offsets"] = tensor(case.cand_offsets, torch.int64, device)
        out["cand_emb"] = tensor(case.cand_emb, dt, device)
        out["request_ts"] = tensor(case.request_ts, torch.int64, device)
    return out
