"""CPU tests of the C-ABI boundary: the library loads, exports every function
declared in include/kda.h, and rejects bad arguments with a status code before
touching the GPU. Only argument combinations that fail validation are passed
here (they return before any CUDA call), so nothing runs on a device.
"""
import ctypes
import os
import re

import pytest

import gated_delta_rule_134_b200 as kda

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    names = []
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names += re.findall(r"\b(kda_[a-z0-9_]+)\s*\(", src)
    return sorted(set(names))


def test_library_exports_every_declared_symbol():
    lib = kda.load()
    names = declared_functions()
    assert "kda_chunk_fwd" in names and "kda_decode_step" in names
    for n in names:
        assert hasattr(lib, n), n


def test_status_strings():
    lib = kda.load()
    for code in range(5):
        s = lib.kda_status_string(code).decode()
        assert s.startswith(kda.STATUS[code])


def _chunk(lib, ptrs, B=1, T=4, H=1, dk=64, dv=64, chunk=64, dtype=1, ws=None, ws_len=0, algo=0):
    q, k, v, la, beta, S0, o, ST = ptrs
    return lib.kda_chunk_fwd_ex(q, k, v, la, beta, S0, o, ST, B, T, H, dk, dv, chunk, dtype, ws, ws_len, algo,
                                None)


GOOD = [ctypes.c_void_p(0x1000 * (i + 1)) for i in range(5)] + [None, ctypes.c_void_p(0x7000), None]


@pytest.mark.parametrize("which", range(5))
def test_chunk_rejects_null_input(which):
    lib = kda.load()
    ptrs = list(GOOD)
    ptrs[which] = None
    assert _chunk(lib, ptrs) == 1


def test_chunk_rejects_null_output():
    lib = kda.load()
    ptrs = list(GOOD)
    ptrs[6] = None
    assert _chunk(lib, ptrs) == 1


def test_chunk_rejects_misaligned():
    lib = kda.load()
    ptrs = list(GOOD)
    ptrs[2] = ctypes.c_void_p(0x3008)
    assert _chunk(lib, ptrs) == 1
    ptrs = list(GOOD)
    ptrs[5] = ctypes.c_void_p(0x9004)  # S0
    assert _chunk(lib, ptrs) == 1


@pytest.mark.parametrize("dk,dv", [(32, 32), (64, 128), (96, 96), (256, 256)])
def test_chunk_rejects_unsupported_head_size(dk, dv):
    lib = kda.load()
    assert _chunk(lib, GOOD, dk=dk, dv=dv) == 2


@pytest.mark.parametrize("chunk", [0, 8, 48, 128])
def test_chunk_rejects_unsupported_chunk(chunk):
    lib = kda.load()
    assert _chunk(lib, GOOD, chunk=chunk) == 2


def test_chunk_rejects_bad_sizes_and_enums():
    lib = kda.load()
    assert _chunk(lib, GOOD, B=-1) == 1
    assert _chunk(lib, GOOD, T=-3) == 1
    assert _chunk(lib, GOOD, dtype=7) == 1
    assert _chunk(lib, GOOD, algo=9) == 1


def test_tc_path_rejects_shapes_it_does_not_cover():
    lib = kda.load()
    assert _chunk(lib, GOOD, dtype=0, dk=128, dv=128, algo=2) == 2   # fp32
    assert _chunk(lib, GOOD, dtype=1, dk=64, dv=64, algo=2) == 2     # d = 64
    assert _chunk(lib, GOOD, dtype=1, dk=128, dv=128, chunk=32, algo=2) == 2


def test_timeout_hook_rejects_bad_budget_and_shapes():
    """The fault-injection hook checks its own arguments before any launch."""
    lib = kda.load()
    q, k, v, la, beta, S0, o, ST = GOOD

    def hook(budget, T=64, dtype=1, dk=128):
        return lib.kda_chunk_fwd_timeout_test(q, k, v, la, beta, S0, o, ST, 1, T, 1, dk, dk, 64, dtype, None, 0,
                                              budget, None)

    assert hook(0) == 1 and hook(-5) == 1 and hook((1 << 31) + 1) == 1   # budget out of range
    assert hook(1 << 20, T=0) == 1                                       # nothing to withhold
    assert hook(1 << 20, dtype=0) == 2                                   # fp32: no tensor-core kernel
    assert hook(1 << 20, dk=64) == 2
    assert hook(1 << 20) == 1                                            # no workspace


def test_workspace_size_is_host_only():
    lib = kda.load()
    assert lib.kda_chunk_fwd_workspace_size(1, 16, 1, 64, 64, 64, 0, 1) == 0   # SIMT needs none
    assert lib.kda_chunk_fwd_workspace_size(1, 16, 1, 48, 48, 64, 0, 0) == 0   # invalid -> 0


def test_decode_rejects_bad_args():
    lib = kda.load()
    p = [ctypes.c_void_p(0x1000 * (i + 1)) for i in range(8)]
    f = lib.kda_decode_step
    for i in range(8):
        pp = list(p)
        pp[i] = None
        assert f(*pp, 2, 2, 128, 128, 1, None) == 1
    pp = list(p)
    pp[5] = ctypes.c_void_p(0x6004)
    assert f(*pp, 2, 2, 128, 128, 1, None) == 1
    assert f(*p, 2, 2, 96, 96, 1, None) == 2
    assert f(*p, 2, 2, 128, 64, 1, None) == 2
    assert f(*p, -1, 2, 128, 128, 1, None) == 1
    assert f(*p, 2, 2, 128, 128, 5, None) == 1


def test_binding_has_no_cpu_fallback():
    torch = pytest.importorskip("torch")
    x = torch.zeros(1, 4, 1, 64)
    b = torch.zeros(1, 4, 1)
    v = torch.zeros(1, 4, 1, 64)
    # CPU tensors are refused before any call into the library: there is no CPU path.
    with pytest.raises(ValueError, match="CUDA tensor"):
        kda.chunk_fwd(x, x, v, x, b)
    with pytest.raises(ValueError, match="CUDA tensor"):
        kda.decode_step(x[:, 0], x[:, 0], v[:, 0], x[:, 0], b[:, 0], torch.zeros(1, 1, 64, 64))


# ---------------------------------------------------------------- variant switches


def _chunk_v(lib, ptrs, erase=1, gate=0, B=1, T=4, H=1, dk=64, dv=64, chunk=64, dtype=1, algo=0):
    q, k, v, la, beta, S0, o, ST = ptrs
    return lib.kda_chunk_fwd_v(q, k, v, la, beta, S0, o, ST, B, T, H, dk, dv, chunk, dtype, erase, gate, None, 0,
                               algo, None)


@pytest.mark.parametrize("erase,gate", [(2, 0), (-1, 0), (1, 3), (0, -1)])
def test_variant_rejects_bad_switches(erase, gate):
    assert _chunk_v(kda.load(), GOOD, erase=erase, gate=gate) == 1


def test_variant_gate_needs_log_alpha():
    lib = kda.load()
    ptrs = list(GOOD)
    ptrs[3] = None
    for gate in (0, 1):
        assert _chunk_v(lib, ptrs, gate=gate) == 1


def test_variant_gate_none_accepts_null_log_alpha():
    # passes pointer validation and stops at the next check (tensor-core
    # algorithm with f32 inputs is unsupported), so nothing is launched
    lib = kda.load()
    ptrs = list(GOOD)
    ptrs[3] = None
    assert _chunk_v(lib, ptrs, gate=2, dtype=0, algo=2) == 2


@pytest.mark.parametrize("erase,gate", [(2, 0), (1, 5)])
def test_decode_variant_rejects_bad_switches(erase, gate):
    lib = kda.load()
    p = [ctypes.c_void_p(0x1000 * (i + 1)) for i in range(8)]
    assert lib.kda_decode_step_v(*p, 2, 1, 64, 64, 1, erase, gate, None) == 1


def test_varlen_rejects_missing_or_misaligned_offsets():
    lib = kda.load()
    q, k, v, la, beta, S0, o, ST = GOOD
    args = lambda cu: (q, k, v, la, beta, S0, o, ST, cu, 2, 8, 1, 64, 64, 64, 1, 1, 0, None, 0, 0, None)
    assert lib.kda_chunk_fwd_varlen(*args(None)) == 1
    assert lib.kda_chunk_fwd_varlen(*args(ctypes.c_void_p(0x5002))) == 1


def test_scan_workspace_sizes():
    """The segment scan keeps B*H*(3P-5) fp32 [128][128] matrices after the
    256-byte status block; it is planned only where its depth in chunk periods
    beats one pass (auto), never for 128 heads (one wave of whole sequences
    already fills 148 SMs). Without a GPU the planner assumes 148 SMs."""
    mat = 128 * 128 * 4
    # 32 heads, 2048 chunks: P = 5 (phase 1 in two waves, phase 3 in one: a depth
    # of 3 x 410 chunks against 2 x 683 for P = 3) -> 10 matrices per head
    assert kda.workspace_size(1, 131072, 32, 128, 128, 64, "bf16", "tc_scan") == 256 + 32 * 10 * mat
    assert kda.workspace_size(1, 131072, 32, 128, 128, 64, "bf16", "auto") == 256 + 32 * 10 * mat
    # 16 heads x 2, 64 chunks, and 32 heads x 1, 32 chunks: short segments, where
    # filling each CTA's pipeline weighs in: P = 3
    assert kda.workspace_size(2, 4096, 16, 128, 128, 64, "bf16", "auto") == 256 + 32 * 4 * mat
    assert kda.workspace_size(1, 2048, 32, 128, 128, 64, "bf16", "auto") == 256 + 32 * 4 * mat
    assert kda.workspace_size(1, 131072, 32, 128, 128, 64, "bf16", "tc") == 256
    assert kda.workspace_size(4, 8192, 32, 128, 128, 64, "bf16", "auto") == 256
    # 2 heads, 65 chunks, forced: P = 32 -> Lc = 3 chunks -> 22 segments
    assert kda.workspace_size(1, 4100, 2, 128, 128, 64, "bf16", "tc_scan") == 256 + 2 * (3 * 22 - 5) * mat
    # forced on 3 chunks: one chunk per segment, P = 3
    assert kda.workspace_size(1, 191, 1, 128, 128, 64, "bf16", "tc_scan") == 256 + 4 * mat
    # too short to split (2 chunks): plain
    assert kda.workspace_size(1, 100, 1, 128, 128, 64, "bf16", "tc_scan") == 256
    assert kda.workspace_size(1, 1000, 1, 128, 128, 64, "bf16", "auto") == 256


def _bwd(lib, ptrs, ws=None, ws_bytes=0, gate=0, erase=1, d=64):
    # q, k, v, log_alpha, beta, S0, dO, dS_T, d_q, d_k, d_v, d_log_alpha, d_beta, d_S0
    return lib.kda_chunk_bwd(*ptrs, 1, 8, 1, d, d, 1, erase, gate, ws, ws_bytes, None)


def _bwd_good():
    p = [ctypes.c_void_p(0x1000 * (i + 1)) for i in range(14)]
    p[5] = p[7] = p[13] = None  # S0, dS_T, d_S0 optional
    return p


def test_bwd_workspace_size():
    d = 128
    # small enough to keep every 8-token chunk's (state, [8][d] delta): 17 chunks per (batch, head)
    assert kda.load().kda_chunk_bwd_workspace_size(2, 130, 3, d, d) == 2 * 3 * 17 * (d * d + 8 * d) * 4
    # beyond 16 GB: one state per 64 tokens plus a ring of 8 (state, delta) slots per (batch, head)
    B, T, H = 1, 131072, 32
    assert kda.load().kda_chunk_bwd_workspace_size(B, T, H, d, d) == B * H * (2048 * d * d + 8 * (d * d + 8 * d)) * 4
    assert kda.load().kda_chunk_bwd_workspace_size(1, 8, 1, 96, 96) == 0


@pytest.mark.parametrize("which", [0, 1, 2, 3, 4, 6, 8, 9, 10, 11, 12])
def test_bwd_rejects_null(which):
    lib = kda.load()
    p = _bwd_good()
    p[which] = None
    ws_bytes = lib.kda_chunk_bwd_workspace_size(1, 8, 1, 64, 64)
    assert _bwd(lib, p, ctypes.c_void_p(0x100000), ws_bytes) == 1


def test_bwd_rejects_small_workspace_and_bad_switches():
    lib = kda.load()
    ws_bytes = lib.kda_chunk_bwd_workspace_size(1, 8, 1, 64, 64)
    assert _bwd(lib, _bwd_good(), ctypes.c_void_p(0x100000), ws_bytes - 4) == 1
    assert _bwd(lib, _bwd_good(), None, 0) == 1
    assert _bwd(lib, _bwd_good(), ctypes.c_void_p(0x100000), ws_bytes, gate=3) == 1
    assert _bwd(lib, _bwd_good(), ctypes.c_void_p(0x100000), ws_bytes, erase=2) == 1
    assert _bwd(lib, _bwd_good(), ctypes.c_void_p(0x100000), ws_bytes, d=96) == 2
    p = _bwd_good()
    p[3] = p[11] = None  # no gate: log_alpha and its gradient may be NULL
    # (valid arguments would launch: check only that validation passes the gate rule by
    # making another required pointer misaligned)
    p[0] = ctypes.c_void_p(0x1001)
    assert _bwd(lib, p, ctypes.c_void_p(0x100000), ws_bytes, gate=2) == 1


def test_bwd_workspace_modes():
    lib = kda.load()
    d = 64
    all_b = 1 * 2 * 10 * (d * d + 8 * d) * 4                 # 77 tokens: 10 chunks of 8
    low_b = 1 * 2 * (2 * d * d + 8 * (d * d + 8 * d)) * 4    # 2 stored states + 8 ring slots
    assert lib.kda_chunk_bwd_workspace_size_ex(1, 77, 2, d, d, 0) == all_b
    assert lib.kda_chunk_bwd_workspace_size_ex(1, 77, 2, d, d, 1) == all_b
    assert lib.kda_chunk_bwd_workspace_size_ex(1, 77, 2, d, d, 2) == low_b
    assert lib.kda_chunk_bwd_workspace_size_ex(1, 77, 2, d, d, 3) == 0
    p = _bwd_good()
    assert lib.kda_chunk_bwd_ex(*p, 1, 8, 1, 64, 64, 1, 1, 0, 7, ctypes.c_void_p(0x100000), 1 << 20, None) == 1


def declared_arity():
    """Number of parameters of every function declared in include/*.h."""
    arity = {}
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            for name, params in re.findall(r"\b(kda_[a-z0-9_]+)\s*\(([^)]*)\)\s*;", src):
                params = params.strip()
                arity[name] = 0 if params in ("", "void") else params.count(",") + 1
    return arity


def test_binding_argtypes_match_declarations():
    """Every argtypes the Python binding sets has the arity of the C
    declaration (a missing or extra argument would shift every later one)."""
    lib = kda.load()
    arity = declared_arity()
    checked = 0
    for name, n in arity.items():
        fn = getattr(lib, name)
        if fn.argtypes is not None:
            assert len(fn.argtypes) == n, (name, len(fn.argtypes), n)
            checked += 1
    assert checked >= 10, checked
