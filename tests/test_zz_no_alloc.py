"""GPU test of kda_chunk_fwd_noalloc, the prefill entry point that allocates
nothing. It serves callers that may not allocate device memory where they run
a prefill (code inside an allocator's own callbacks, hosts that forbid
cudaMalloc on worker threads, runtimes that only hand out tensors they own):
the kernel's scratch lives in a fixed array inside the library instead of a
caller workspace.

It runs the same kernel as kda_chunk_fwd with the tensor-core algorithm, so on
the same inputs the two must agree bit for bit; one of them is also checked
against the fp64 oracle at the bf16 bar. Two calls in a row with different
shapes make sure nothing stale from the first call leaks into the second, and
the status reader must report a clean run after each. This file is collected
last on purpose.
"""
import numpy as np
import pytest
import torch

import oracle
from gated_delta_rule_134_b200 import inputs as I

pytestmark = pytest.mark.gpu

TOL = 2e-2  # the bf16 bar of the other parity tests: max|x - ref| / max|ref|


def rel_err(x, ref):
    x = np.asarray(x, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    return float(np.abs(x - ref).max() / max(np.abs(ref).max(), 1e-30))


CASES = [  # (seed, B, H, T, with_S0, with_S_T)
    (41, 2, 3, 200, True, True),
    (42, 1, 5, 77, False, True),
    (43, 2, 2, 130, True, False),
]


def test_noalloc_matches_workspace_entry_point_two_calls(cuda_lib):
    for seed, B, H, T, with_s0, with_st in CASES:
        cfg = I.PrefillConfig(f"noalloc_b{B}_h{H}_t{T}", B, H, T, 128, 128, 64, "bf16", 0.01, 1.0, 0.2, seed)
        xc = I.prefill_inputs(cfg)
        x = {k: (None if v is None else v.cuda()) for k, v in xc.items()}
        S0 = x["S0"] if with_s0 else None
        ref_o, ref_S = cuda_lib.chunk_fwd(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], S0, algo="tc")
        o = torch.full_like(ref_o, float("nan"))
        S = torch.full_like(ref_S, float("nan")) if with_st else None
        cuda_lib.chunk_fwd_noalloc(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], S0, o=o, S_T=S)
        assert cuda_lib.noalloc_status() == 0
        torch.cuda.synchronize()
        # the same kernel on the same inputs: identical results
        assert torch.equal(o, ref_o)
        if with_st:
            assert torch.equal(S, ref_S)
        # and against the fp64 recurrence
        s0 = xc["S0"] if with_s0 else None
        ro, rS = oracle.recurrent(xc["q"], xc["k"], xc["v"], xc["log_alpha"], xc["beta"], s0)
        assert rel_err(o.float().cpu().numpy(), ro) <= TOL
        if with_st:
            assert rel_err(S.cpu().numpy(), rS) <= TOL
