"""GPU test of kda_chunk_fwd_noalloc, the prefill entry point that allocates
nothing (for callers that may not allocate device memory where they run a
prefill). Its results must match kda_chunk_fwd's on the same inputs, for two
calls in a row with different inputs, so that nothing stale from the first
call leaks into the second. This file is collected last on purpose.
"""
import numpy as np
import pytest
import torch

from gated_delta_rule_134_b200 import inputs as I

pytestmark = pytest.mark.gpu

TOL = 2e-2  # the bf16 bar used by the other parity tests


def rel_err(x, ref):
    x = x.float().cpu().numpy().astype(np.float64)
    ref = ref.float().cpu().numpy().astype(np.float64)
    return float(np.abs(x - ref).max() / max(np.abs(ref).max(), 1e-30))


def test_noalloc_matches_workspace_entry_point_two_calls(cuda_lib):
    for seed, (B, H, T) in ((41, (2, 3, 200)), (42, (1, 5, 77))):
        cfg = I.PrefillConfig(f"noalloc_b{B}_h{H}_t{T}", B, H, T, 128, 128, 64, "bf16", 0.01, 1.0, 0.2, seed)
        x = {k: (None if v is None else v.cuda()) for k, v in I.prefill_inputs(cfg).items()}
        ref_o, ref_S = cuda_lib.chunk_fwd(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], x["S0"], algo="tc")
        o = torch.full_like(ref_o, float("nan"))
        S = torch.full_like(ref_S, float("nan"))
        cuda_lib.chunk_fwd_noalloc(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], x["S0"], o=o, S_T=S)
        torch.cuda.synchronize()
        assert torch.isfinite(o.float()).all() and torch.isfinite(S).all()
        assert rel_err(o, ref_o) <= TOL
        assert rel_err(S, ref_S) <= TOL
