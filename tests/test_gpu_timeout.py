"""GPU test of the device-side timeout path of the tensor-core prefill.

The kernel's warps hand work to one another through shared-memory barriers,
and every wait on one is bounded: when it runs out the kernel records
KDA_ERR_TIMEOUT in the workspace, skips its later waits, waits (bounded) for
its own copies in flight and returns, so the context stays usable. Here the
test hook withholds the first k/q tile load of every CTA and shortens the
budget to 2^20 SM cycles (about half a millisecond), so the first wait on that
tile expires for real. The test checks that the status word says so, that the
call comes back well within a second, and that a normal call afterwards on the
same stream and workspace is parity-green against the fp64 oracle.
"""
import time

import numpy as np
import pytest
import torch

import oracle
from gated_delta_rule_134_b200 import inputs as I

pytestmark = pytest.mark.gpu

TOL = 2e-2           # the bf16 bar of the other parity tests: max|x - ref| / max|ref|
BUDGET = 1 << 20     # SM cycles per wait in the faulted launch
KDA_OK, KDA_ERR_TIMEOUT = 0, 4


def rel_err(x, ref):
    x = np.asarray(x, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    return float(np.abs(x - ref).max() / max(np.abs(ref).max(), 1e-30))


@pytest.mark.parametrize("B,H,T", [(1, 2, 256), (2, 3, 130)])
def test_withheld_load_times_out_then_next_call_is_clean(cuda_lib, B, H, T):
    cfg = I.PrefillConfig(f"timeout_b{B}_h{H}_t{T}", B, H, T, 128, 128, 64, "bf16", 0.01, 1.0, 0.2, 77 + T)
    xc = I.prefill_inputs(cfg)
    x = {k: (None if v is None else v.cuda()) for k, v in xc.items()}
    stream = torch.cuda.Stream()
    ws = torch.zeros(cuda_lib.workspace_size(B, T, H, 128, 128, 64, "bf16", "tc"), dtype=torch.uint8,
                     device="cuda")
    o = torch.empty(B, T, H, 128, dtype=torch.bfloat16, device="cuda")
    S = torch.empty(B, H, 128, 128, dtype=torch.float32, device="cuda")
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        t0 = time.perf_counter()
        cuda_lib.chunk_fwd_timeout_test(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], x["S0"], o=o, S_T=S,
                                        workspace=ws, wait_budget_cycles=BUDGET, stream=stream)
        st = cuda_lib.workspace_status(ws, stream=stream)   # synchronises the stream
        elapsed = time.perf_counter() - t0
    assert st == KDA_ERR_TIMEOUT
    assert elapsed < 1.0, elapsed
    # the context is intact: a normal call on the same stream and workspace
    with torch.cuda.stream(stream):
        o2, S2 = cuda_lib.chunk_fwd(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], x["S0"], algo="tc",
                                    workspace=ws, stream=stream)
        assert cuda_lib.workspace_status(ws, stream=stream) == KDA_OK
    torch.cuda.synchronize()
    ro, rS = oracle.recurrent(xc["q"], xc["k"], xc["v"], xc["log_alpha"], xc["beta"], xc["S0"])
    assert rel_err(o2.float().cpu().numpy(), ro) <= TOL
    assert rel_err(S2.cpu().numpy(), rS) <= TOL
