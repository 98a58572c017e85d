"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle on the
same seeded inputs. Error metric: max|x - ref| / max|ref| over the compared
elements, separately for o and for the final state. Bars: 1e-4 for fp32
inputs, 2e-2 for bf16 inputs with fp32 state/accumulation.

bf16 workloads hand the oracle the same bf16-rounded values (upcast to fp64),
so the measured error is the kernels' own.
"""
import numpy as np
import pytest
import torch

import oracle
from gated_delta_rule_134_b200 import inputs as I

pytestmark = pytest.mark.gpu

TOL = {"f32": 1e-4, "bf16": 2e-2}


def rel_err(x, ref):
    x = np.asarray(x, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    den = np.abs(ref).max()
    return float(np.abs(x - ref).max() / (den if den > 0 else 1.0))


def to_dev(d):
    return {k: (None if v is None else v.cuda()) for k, v in d.items()}


def algos_for(cfg):
    out = ["simt"]
    if cfg.dtype == "bf16" and cfg.dk == 128 and cfg.dv == 128 and cfg.C == 64:
        out.append("tc")
    return out


def small_cfg(dtype, d, C, T, B=2, H=3, la=(0.01, 1.0), s0=0.3, seed=7):
    return I.PrefillConfig(f"small_{dtype}_{d}_{C}_{T}", B, H, T, d, d, C, dtype, la[0], la[1], s0, seed)


def check_prefill(kda, cfg, algo, heads=None):
    x = I.prefill_inputs(cfg)
    xd = to_dev(x)
    o, ST = kda.chunk_fwd(xd["q"], xd["k"], xd["v"], xd["log_alpha"], xd["beta"], xd["S0"], chunk=cfg.C, algo=algo)
    torch.cuda.synchronize()
    if heads is None:
        ref_o, ref_S = oracle.recurrent(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], x["S0"])
        got_o, got_S = o.float().cpu().numpy(), ST.cpu().numpy()
    else:
        xs = I.prefill_inputs(cfg, heads=heads)
        ref_o, ref_S = oracle.recurrent(xs["q"], xs["k"], xs["v"], xs["log_alpha"], xs["beta"], xs["S0"])
        oc, Sc = o.float().cpu(), ST.cpu()
        got_o = np.stack([oc[b, :, h].numpy() for b, h in heads])[:, :, None]
        got_S = np.stack([Sc[b, h].numpy() for b, h in heads])[:, None]
    eo, es = rel_err(got_o, ref_o), rel_err(got_S, ref_S)
    print(f"PARITY {cfg.name} algo={algo} o={eo:.3e} S_T={es:.3e} bar={TOL[cfg.dtype]:.0e}")
    assert np.isfinite(got_o).all() and np.isfinite(got_S).all()
    assert eo <= TOL[cfg.dtype] and es <= TOL[cfg.dtype], (cfg.name, algo, eo, es)
    return eo, es


# ---------------------------------------------------------------- prefill, small


@pytest.mark.parametrize("T", [1, 17, 64, 65, 130, 333])
@pytest.mark.parametrize("C", [16, 32, 64])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_prefill_small_simt(cuda_lib, dtype, d, C, T):
    check_prefill(cuda_lib, small_cfg(dtype, d, C, T), "simt")


@pytest.mark.parametrize("s0", [0.0, 0.3])
@pytest.mark.parametrize("T", [1, 17, 63, 64, 65, 130, 333, 1000])
def test_prefill_small_tc(cuda_lib, T, s0):
    check_prefill(cuda_lib, small_cfg("bf16", 128, 64, T, s0=s0), "tc")


@pytest.mark.parametrize("algo", ["simt", "tc"])
@pytest.mark.parametrize("la", [(1.0, 8.0), (0.0, 0.0), (0.0, 1e-4)])
def test_prefill_decay_extremes(cuda_lib, algo, la):
    # strong decay (exercises the overflow-safe path of the tensor-core kernel),
    # no decay at all, and nearly none
    check_prefill(cuda_lib, small_cfg("bf16", 128, 64, 200, la=la), algo)


@pytest.mark.parametrize("la", [(1.0, 2.0), (1.5, 3.0)])
def test_prefill_tc_mid_reference_tier(cuda_lib, la):
    # a decay of 64-190 per chunk: the chunk-start reference fails its guard, the
    # G_last / 2 reference takes chunks up to 160 (stronger ones: the exact path);
    # ragged tail, entry state
    check_prefill(cuda_lib, small_cfg("bf16", 128, 64, 333, la=la, seed=37), "tc")


@pytest.mark.parametrize("algo", ["simt", "tc"])
def test_prefill_many_heads_small(cuda_lib, algo):
    # more (b, h) pairs than SMs, ragged tail
    check_prefill(cuda_lib, small_cfg("bf16", 128, 64, 77, B=3, H=70, seed=9), algo)


# ---------------------------------------------------------------- prefill, edge cases


@pytest.mark.parametrize("algo", ["simt", "tc"])
def test_prefill_empty_sequence_copies_state(cuda_lib, algo):
    cfg = small_cfg("bf16", 128, 64, 0)
    x = to_dev(I.prefill_inputs(cfg))
    o, ST = cuda_lib.chunk_fwd(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], x["S0"], algo=algo)
    torch.cuda.synchronize()
    assert o.numel() == 0
    assert torch.equal(ST, x["S0"])
    o, ST = cuda_lib.chunk_fwd(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], None, algo=algo)
    assert torch.count_nonzero(ST).item() == 0


def test_prefill_empty_batch(cuda_lib):
    z = torch.empty(0, 5, 2, 128, dtype=torch.bfloat16, device="cuda")
    o, ST = cuda_lib.chunk_fwd(z, z, z, z, torch.empty(0, 5, 2, dtype=torch.bfloat16, device="cuda"))
    assert o.shape == (0, 5, 2, 128) and ST.shape == (0, 2, 128, 128)


@pytest.mark.parametrize("algo", ["simt", "tc"])
def test_prefill_state_in_place_and_chaining(cuda_lib, algo):
    cfg = small_cfg("bf16", 128, 64, 300)
    x = to_dev(I.prefill_inputs(cfg))
    o_full, S_full = cuda_lib.chunk_fwd(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], x["S0"], algo=algo)
    S = x["S0"].clone()
    outs = []
    for a, b in [(0, 100), (100, 101), (101, 300)]:
        sl = {kk: x[kk][:, a:b].contiguous() for kk in ("q", "k", "v", "log_alpha", "beta")}
        o, _ = cuda_lib.chunk_fwd(sl["q"], sl["k"], sl["v"], sl["log_alpha"], sl["beta"], S, S_T=S, algo=algo)
        outs.append(o)
    torch.cuda.synchronize()
    assert rel_err(torch.cat(outs, 1).float().cpu(), o_full.float().cpu()) < 2e-2
    assert rel_err(S.cpu(), S_full.cpu()) < 2e-2


@pytest.mark.parametrize("algo", ["simt", "tc"])
def test_prefill_deterministic(cuda_lib, algo):
    cfg = small_cfg("bf16", 128, 64, 257)
    x = to_dev(I.prefill_inputs(cfg))
    r1 = cuda_lib.chunk_fwd(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], x["S0"], algo=algo)
    r2 = cuda_lib.chunk_fwd(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], x["S0"], algo=algo)
    torch.cuda.synchronize()
    assert torch.equal(r1[0], r2[0]) and torch.equal(r1[1], r2[1])


@pytest.mark.parametrize("la", [(0.001, 0.1), (0.01, 1.0)])
def test_prefill_tc_repeat_every_head(cuda_lib, la):
    """The tensor-core kernel overlaps the preparation of chunk n+1 with the
    state-dependent work of chunk n; a missing hand-over between the two shows
    up as timing-dependent errors in isolated chunks. Repeat runs of a
    many-chunk, many-CTA case must agree bit for bit, and every head must
    match the oracle (weak decay keeps errors of the carried state visible)."""
    cfg = small_cfg("bf16", 128, 64, 1536, B=2, H=16, la=la, s0=0.1, seed=21)
    x = I.prefill_inputs(cfg)
    xd = to_dev(x)
    runs = [cuda_lib.chunk_fwd(xd["q"], xd["k"], xd["v"], xd["log_alpha"], xd["beta"], xd["S0"], algo="tc")
            for _ in range(3)]
    torch.cuda.synchronize()
    for o, ST in runs[1:]:
        assert torch.equal(o, runs[0][0]) and torch.equal(ST, runs[0][1])
    ref_o, ref_S = oracle.recurrent(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], x["S0"])
    eo, es = rel_err(runs[0][0].float().cpu().numpy(), ref_o), rel_err(runs[0][1].cpu().numpy(), ref_S)
    print(f"PARITY repeat_every_head la={la} o={eo:.3e} S_T={es:.3e} bar={TOL['bf16']:.0e}")
    assert eo <= TOL["bf16"] and es <= TOL["bf16"], (eo, es)


def test_prefill_no_final_state(cuda_lib):
    cfg = small_cfg("f32", 64, 64, 70)
    x = to_dev(I.prefill_inputs(cfg))
    o, ST = cuda_lib.chunk_fwd(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], x["S0"],
                               output_final_state=False)
    assert ST is None
    ref, _ = oracle.recurrent(*[I.prefill_inputs(cfg)[kk] for kk in ("q", "k", "v", "log_alpha", "beta", "S0")])
    assert rel_err(o.cpu().numpy(), ref) < 1e-4


# ---------------------------------------------------------------- prefill, full-size workloads


def test_prefill_small_f32_full(cuda_lib):
    check_prefill(cuda_lib, I.SMALL_F32, "auto")


@pytest.mark.parametrize("algo", ["auto", "tc", "simt"])
def test_prefill_b2_h16_t4k(cuda_lib, algo):
    check_prefill(cuda_lib, I.B2_H16_T4K, algo, heads=[(0, 0), (0, 7), (1, 3), (1, 15)])


def test_prefill_b4_h32_t8k(cuda_lib):
    check_prefill(cuda_lib, I.B4_H32_T8K, "auto", heads=[(0, 0), (0, 31), (1, 5), (2, 17), (3, 2), (3, 30)])


@pytest.mark.parametrize("algo", ["auto", "tc"])
def test_prefill_b1_h32_t128k(cuda_lib, algo):
    # auto takes the segment scan here (32 heads, 2048 chunks)
    check_prefill(cuda_lib, I.B1_H32_T128K, algo, heads=[(0, 0), (0, 13), (0, 31)])


# ---------------------------------------------------------------- decode


@pytest.mark.parametrize("inplace", [True, False])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_decode_small_chain(cuda_lib, dtype, d, inplace):
    cfg = I.DecodeConfig("decode_small", 5, 3, d, d, 30, dtype, 0.001, 0.5, 0.1, 3)
    S_ref = I.decode_state(cfg).double().numpy()
    S = I.decode_state(cfg).cuda()
    for step in range(cfg.steps):
        x = I.decode_step_inputs(cfg, step)
        xd = to_dev(x)
        S_out = S if inplace else torch.empty_like(S)
        o, S_new = cuda_lib.decode_step(xd["q"], xd["k"], xd["v"], xd["log_alpha"], xd["beta"], S, S_out=S_out)
        o_ref, S_ref = oracle.decode_step(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], S_ref)
        assert rel_err(o.float().cpu().numpy(), o_ref) <= TOL[dtype]
        S = S_new
    torch.cuda.synchronize()
    assert rel_err(S.cpu().numpy(), S_ref) <= TOL[dtype]


def test_decode_full_first_step_all_heads(cuda_lib):
    cfg = I.DECODE_N256_H32
    S0 = I.decode_state(cfg)
    x = I.decode_step_inputs(cfg, 0)
    xd = to_dev(x)
    S = S0.cuda()
    o, S = cuda_lib.decode_step(xd["q"], xd["k"], xd["v"], xd["log_alpha"], xd["beta"], S)
    o_ref, S_ref = oracle.decode_step(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], S0)
    assert rel_err(o.float().cpu().numpy(), o_ref) <= TOL["bf16"]
    assert rel_err(S.cpu().numpy(), S_ref) <= TOL["bf16"]


def test_decode_full_1000_steps_sampled_heads(cuda_lib):
    """All 1000 chained in-place steps on the full [256,32,128,128] state; the
    oracle follows 64 seeded heads (heads are independent, so this is exact
    for the sample)."""
    cfg = I.DECODE_N256_H32
    rng = np.random.default_rng(1234)
    idx = rng.choice(cfg.N * cfg.H, size=64, replace=False)
    heads = [(int(i) // cfg.H, int(i) % cfg.H) for i in idx]
    nn = torch.tensor([n for n, _ in heads])
    hh = torch.tensor([h for _, h in heads])
    S_full = I.decode_state(cfg)
    S_ref = S_full[nn, hh].double().numpy()[:, None]
    S = S_full.cuda()
    del S_full
    worst = 0.0
    for step in range(cfg.steps):
        x = I.decode_step_inputs(cfg, step)
        xd = to_dev(x)
        o, S = cuda_lib.decode_step(xd["q"], xd["k"], xd["v"], xd["log_alpha"], xd["beta"], S)
        xs = {kk: x[kk][nn, hh][:, None] for kk in x}
        o_ref, S_ref = oracle.decode_step(xs["q"], xs["k"], xs["v"], xs["log_alpha"], xs["beta"], S_ref)
        worst = max(worst, rel_err(o[nn.cuda(), hh.cuda()].float().cpu().numpy()[:, None], o_ref))
    torch.cuda.synchronize()
    assert worst <= TOL["bf16"]
    assert rel_err(S[nn.cuda(), hh.cuda()].cpu().numpy()[:, None], S_ref) <= TOL["bf16"]


# ---------------------------------------------------------------- variants (erase / gate switches)

VARIANTS = [(True, "scalar"), (True, "none"), (False, "channel"), (False, "scalar"), (False, "none")]


def _variant_inputs(cfg, gate):
    x = I.prefill_inputs(cfg)
    la = x["log_alpha"]
    x["log_alpha"] = {"channel": la, "scalar": la[..., 0].contiguous(), "none": None}[gate]
    return x


def check_variant(kda, cfg, algo, erase, gate):
    x = _variant_inputs(cfg, gate)
    xd = to_dev(x)
    o, ST = kda.chunk_fwd(xd["q"], xd["k"], xd["v"], xd["log_alpha"], xd["beta"], xd["S0"], chunk=cfg.C, algo=algo,
                          erase=erase, gate=gate)
    torch.cuda.synchronize()
    ref_o, ref_S = oracle.recurrent(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], x["S0"], erase=erase,
                                    gate=gate)
    eo, es = rel_err(o.float().cpu().numpy(), ref_o), rel_err(ST.cpu().numpy(), ref_S)
    print(f"PARITY variant erase={int(erase)} gate={gate} {cfg.name} algo={algo} o={eo:.3e} S_T={es:.3e} "
          f"bar={TOL[cfg.dtype]:.0e}")
    assert np.isfinite(o.float().cpu().numpy()).all() and np.isfinite(ST.cpu().numpy()).all()
    assert eo <= TOL[cfg.dtype] and es <= TOL[cfg.dtype], (cfg.name, algo, erase, gate, eo, es)


@pytest.mark.parametrize("erase,gate", VARIANTS)
@pytest.mark.parametrize("algo", ["simt", "tc"])
@pytest.mark.parametrize("la", [(0.01, 1.0), (0.001, 0.1)])
def test_prefill_variants_bf16(cuda_lib, algo, erase, gate, la):
    check_variant(cuda_lib, small_cfg("bf16", 128, 64, 200, la=la, s0=0.3, seed=31), algo, erase, gate)


@pytest.mark.parametrize("erase,gate", VARIANTS)
def test_prefill_variants_f32(cuda_lib, erase, gate):
    check_variant(cuda_lib, small_cfg("f32", 64, 32, 97, s0=0.3, seed=32), "simt", erase, gate)


@pytest.mark.parametrize("erase,gate", [(True, "scalar"), (False, "channel")])
def test_prefill_variants_tc_extreme_decay(cuda_lib, erase, gate):
    # decays up to e^-6 per token: the guard sends chunks down the exact path
    check_variant(cuda_lib, small_cfg("bf16", 128, 64, 150, la=(0.5, 6.0), seed=33), "tc", erase, gate)


@pytest.mark.parametrize("erase,gate", VARIANTS)
def test_prefill_variants_tc_mid_reference_tier(cuda_lib, erase, gate):
    # decays of 64-128 per chunk: every full chunk takes the G_last / 2 reference
    check_variant(cuda_lib, small_cfg("bf16", 128, 64, 333, la=(1.0, 2.0), seed=38), "tc", erase, gate)


@pytest.mark.parametrize("erase,gate", VARIANTS)
def test_prefill_variants_tc_many_chunks(cuda_lib, erase, gate):
    check_variant(cuda_lib, small_cfg("bf16", 128, 64, 1536, B=2, H=16, la=(0.001, 0.1), s0=0.1, seed=34), "tc",
                  erase, gate)


@pytest.mark.parametrize("erase,gate", VARIANTS)
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_decode_variants_chain(cuda_lib, erase, gate, dtype):
    cfg = I.DecodeConfig("decode_variant", 3, 5, 128, 128, 6, dtype, 0.01, 1.0, 0.2, 35)
    S = I.decode_state(cfg)
    Sd = S.cuda()
    S_ref = S.double().numpy()
    for step in range(cfg.steps):
        x = I.decode_step_inputs(cfg, step)
        la = x["log_alpha"]
        x["log_alpha"] = {"channel": la, "scalar": la[..., 0].contiguous(), "none": None}[gate]
        xd = to_dev(x)
        o, Sd = cuda_lib.decode_step(xd["q"], xd["k"], xd["v"], xd["log_alpha"], xd["beta"], Sd, erase=erase,
                                     gate=gate)
        ref_o, S_ref = oracle.decode_step(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], S_ref, erase=erase,
                                          gate=gate)
        torch.cuda.synchronize()
        assert rel_err(o.float().cpu().numpy(), ref_o) <= TOL[dtype]
    assert rel_err(Sd.cpu().numpy(), S_ref) <= TOL[dtype]


# ---------------------------------------------------------------- packed variable-length sequences


def _gate_view(la, gate):
    return {"channel": la, "scalar": None if la is None else la[..., 0].contiguous(), "none": None}[gate]


def check_varlen(kda, cfg, lengths, algo, erase=True, gate="channel"):
    x = I.varlen_inputs(cfg, lengths)
    x["log_alpha"] = _gate_view(x["log_alpha"], gate)
    xd = to_dev(x)
    o, ST = kda.chunk_fwd_varlen(xd["q"], xd["k"], xd["v"], xd["log_alpha"], xd["beta"], xd["cu_seqlens"], xd["S0"],
                                 chunk=cfg.C, algo=algo, erase=erase, gate=gate)
    torch.cuda.synchronize()
    ref_o, ref_S = oracle.recurrent_varlen(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], x["cu_seqlens"],
                                           x["S0"], erase=erase, gate=gate)
    got_o, got_S = o.float().cpu().numpy(), ST.cpu().numpy()
    assert np.isfinite(got_o).all() and np.isfinite(got_S).all()
    eo = rel_err(got_o, ref_o) if got_o.size else 0.0
    es = rel_err(got_S, ref_S)
    print(f"PARITY varlen {cfg.name} N={len(lengths)} total={sum(lengths)} algo={algo} erase={int(erase)} "
          f"gate={gate} o={eo:.3e} S_T={es:.3e}")
    assert eo <= TOL[cfg.dtype] and es <= TOL[cfg.dtype], (lengths, algo, eo, es)
    return o, ST


VARLEN_MIXES = [[0, 1, 63, 64, 65, 200], [300], [5, 0, 0, 129], [128, 1, 0], [0]]


@pytest.mark.parametrize("lengths", VARLEN_MIXES)
@pytest.mark.parametrize("algo", ["simt", "tc"])
def test_varlen_mixes_bf16(cuda_lib, algo, lengths):
    check_varlen(cuda_lib, small_cfg("bf16", 128, 64, 0, H=3, s0=0.3, seed=41), lengths, algo)


@pytest.mark.parametrize("C", [16, 32, 64])
def test_varlen_f32_simt(cuda_lib, C):
    check_varlen(cuda_lib, small_cfg("f32", 64, C, 0, H=2, s0=0.3, seed=42), [17, 0, 33, 64, 1, 90], "simt")


@pytest.mark.parametrize("algo", ["simt", "tc"])
def test_varlen_many_sequences(cuda_lib, algo):
    lengths = I.varlen_lengths(40, 150, seed=43, zero_frac=0.1)
    check_varlen(cuda_lib, small_cfg("bf16", 128, 64, 0, H=4, s0=0.2, seed=43), lengths, algo)


@pytest.mark.parametrize("erase,gate", VARIANTS)
@pytest.mark.parametrize("algo", ["simt", "tc"])
def test_varlen_variants(cuda_lib, algo, erase, gate):
    check_varlen(cuda_lib, small_cfg("bf16", 128, 64, 0, H=2, s0=0.3, seed=44), [70, 0, 129, 3], algo, erase, gate)


def test_varlen_tc_extreme_decay(cuda_lib):
    # strong decay sends chunks down the exact path; tails end mid-chunk
    check_varlen(cuda_lib, small_cfg("bf16", 128, 64, 0, H=2, la=(0.5, 6.0), seed=45), [100, 37, 64, 190], "tc")


@pytest.mark.parametrize("algo", ["simt", "tc"])
def test_varlen_equal_lengths_match_dense(cuda_lib, algo):
    """Packing B equal-length sequences must give exactly the dense [B, T] result:
    the same kernel does the same arithmetic on the same tokens."""
    cfg = I.B2_H16_T4K if algo == "tc" else small_cfg("bf16", 128, 64, 777, B=3, H=4, s0=0.3, seed=46)
    x = to_dev(I.prefill_inputs(cfg))
    o_d, S_d = cuda_lib.chunk_fwd(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], x["S0"], chunk=64, algo=algo)
    pack = lambda t: t.reshape((-1,) + tuple(t.shape[2:]))
    cu = torch.arange(0, cfg.B + 1, dtype=torch.int32, device="cuda") * cfg.T
    o_v, S_v = cuda_lib.chunk_fwd_varlen(pack(x["q"]), pack(x["k"]), pack(x["v"]), pack(x["log_alpha"]),
                                         pack(x["beta"]), cu, x["S0"], chunk=64, algo=algo)
    torch.cuda.synchronize()
    assert torch.equal(pack(o_d), o_v) and torch.equal(S_d, S_v)


def test_varlen_full_size_sampled(cuda_lib):
    """A packed batch of 24 sequences (about 35K tokens, H32 d128, strong
    decay) with mixed lengths; sampled (sequence, head) slices against the
    oracle."""
    lengths = I.varlen_lengths(24, 1365, seed=47, zero_frac=0.05)
    cfg = I.B4_H32_T8K.replace(s0_std=0.05, seed=47)
    x = I.varlen_inputs(cfg, lengths)
    xd = to_dev(x)
    o, ST = cuda_lib.chunk_fwd_varlen(xd["q"], xd["k"], xd["v"], xd["log_alpha"], xd["beta"], xd["cu_seqlens"],
                                      xd["S0"], chunk=64, algo="auto")
    torch.cuda.synchronize()
    cu = x["cu_seqlens"].tolist()
    rng = np.random.default_rng(47)
    worst = 0.0
    for n in rng.choice(len(lengths), 6, replace=False):
        h = int(rng.integers(cfg.H))
        a, b = cu[n], cu[n + 1]
        sl = lambda t: t[a:b, h:h + 1][None]
        s0 = None if x["S0"] is None else x["S0"][n:n + 1, h:h + 1]
        ref_o, ref_S = oracle.recurrent(sl(x["q"]), sl(x["k"]), sl(x["v"]), sl(x["log_alpha"]), sl(x["beta"]), s0)
        if b > a:
            worst = max(worst, rel_err(o[a:b, h].float().cpu().numpy()[None, :, None], ref_o))
        worst = max(worst, rel_err(ST[n, h].cpu().numpy()[None, None], ref_S))
    print(f"PARITY varlen full-size sampled worst={worst:.3e}")
    assert worst <= TOL["bf16"]


# ---------------------------------------------------------------- chunk-parallel segment scan (tc_scan)


@pytest.mark.parametrize("B,H,T,s0", [(2, 3, 1000, 0.3), (1, 1, 777, 0.0), (1, 2, 4100, 0.2), (3, 2, 384, 0.3),
                                      (1, 1, 191, 0.3), (1, 1, 100, 0.3)])
def test_scan_small(cuda_lib, B, H, T, s0):
    """Segments of 2+ chunks, a ragged last segment, many segments in the scan
    chain (T=4100 on 2 heads: 22 segments), one-chunk segments (T=191) and the
    plain fallback (T=100, two chunks)."""
    check_prefill(cuda_lib, small_cfg("bf16", 128, 64, T, B=B, H=H, s0=s0, seed=60 + T), "tc_scan")


@pytest.mark.parametrize("erase,gate", VARIANTS)
def test_scan_variants(cuda_lib, erase, gate):
    check_variant(cuda_lib, small_cfg("bf16", 128, 64, 1100, B=1, H=2, s0=0.3, seed=61), "tc_scan", erase, gate)


@pytest.mark.parametrize("algo", ["tc_scan", "auto"])
def test_scan_weak_decay(cuda_lib, algo):
    """Weak decay over short segments: every segment's output depends on its
    entry state, so errors in the maps or the scan would show everywhere."""
    check_prefill(cuda_lib, small_cfg("bf16", 128, 64, 3000, B=1, H=2, la=(0.0001, 0.005), s0=0.3, seed=66), algo)


def test_scan_extreme_decay(cuda_lib):
    # strong decay: chunks take the exact path inside the segment runs too
    check_prefill(cuda_lib, small_cfg("bf16", 128, 64, 900, B=1, H=2, la=(0.5, 6.0), s0=0.3, seed=62), "tc_scan")


def test_scan_state_aliasing(cuda_lib):
    """S_T may alias S0: segment 0 reads S0 in the first launch, the last
    segment writes S_T in the last one."""
    cfg = small_cfg("bf16", 128, 64, 1000, B=1, H=3, s0=0.3, seed=63)
    x = I.prefill_inputs(cfg)
    xd = to_dev(x)
    S = xd["S0"].clone()
    o, ST = cuda_lib.chunk_fwd(xd["q"], xd["k"], xd["v"], xd["log_alpha"], xd["beta"], S, S_T=S, algo="tc_scan")
    torch.cuda.synchronize()
    ref_o, ref_S = oracle.recurrent(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], x["S0"])
    assert rel_err(o.float().cpu().numpy(), ref_o) <= TOL["bf16"]
    assert rel_err(S.cpu().numpy(), ref_S) <= TOL["bf16"]


def test_scan_deterministic(cuda_lib):
    cfg = small_cfg("bf16", 128, 64, 2000, B=1, H=4, s0=0.3, seed=64)
    x = to_dev(I.prefill_inputs(cfg))
    outs = [cuda_lib.chunk_fwd(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], x["S0"], algo="tc_scan")
            for _ in range(3)]
    torch.cuda.synchronize()
    for o, ST in outs[1:]:
        assert torch.equal(o, outs[0][0]) and torch.equal(ST, outs[0][1])


def test_scan_varlen_unsupported(cuda_lib):
    x = to_dev(I.varlen_inputs(small_cfg("bf16", 128, 64, 0, H=1, seed=65), [100, 200]))
    with pytest.raises(RuntimeError):
        cuda_lib.chunk_fwd_varlen(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], x["cu_seqlens"], x["S0"],
                                  algo="tc_scan")


# ---------------------------------------------------------------- backward (kda_chunk_bwd)


BWD_NAMES = ("dq", "dk", "dv", "dlog_alpha", "dbeta", "dS0")


def check_bwd(kda, cfg, erase=True, gate="channel", with_dST=True, memory="auto"):
    x = _variant_inputs(cfg, gate)
    c = I.bwd_cotangents(cfg, with_dST)
    xd, cd = to_dev(x), to_dev(c)
    g = kda.chunk_bwd(xd["q"], xd["k"], xd["v"], xd["log_alpha"], xd["beta"], xd["S0"], cd["dO"], cd["dST"],
                      erase=erase, gate=gate, memory=memory)
    torch.cuda.synchronize()
    ref = oracle.recurrent_bwd(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], x["S0"], c["dO"], c["dST"],
                               erase=erase, gate=gate)
    errs = {}
    for n in BWD_NAMES:
        if ref[n] is None:
            assert g[n] is None
            continue
        got = g[n].float().cpu().numpy()
        assert np.isfinite(got).all(), n
        errs[n] = rel_err(got, ref[n]) if got.size else 0.0
    print(f"PARITY bwd {cfg.name} erase={int(erase)} gate={gate} memory={memory} " + " ".join(f"{n}={e:.2e}" for n, e in errs.items()))
    for n, e in errs.items():
        assert e <= TOL[cfg.dtype], (cfg.name, erase, gate, n, e)
    return g


@pytest.mark.parametrize("T", [1, 9, 64, 77, 200])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_bwd_small(cuda_lib, dtype, d, T):
    check_bwd(cuda_lib, small_cfg(dtype, d, 64, T, B=2, H=2, s0=0.3, seed=70 + T))


@pytest.mark.parametrize("erase,gate", VARIANTS)
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_bwd_variants(cuda_lib, dtype, erase, gate):
    d = 64 if dtype == "f32" else 128
    check_bwd(cuda_lib, small_cfg(dtype, d, 64, 150, B=1, H=2, s0=0.3, seed=71), erase, gate)


@pytest.mark.parametrize("la", [(0.5, 6.0), (0.0, 1e-4)])
def test_bwd_decay_extremes(cuda_lib, la):
    check_bwd(cuda_lib, small_cfg("f32", 128, 64, 130, B=1, H=2, la=la, s0=0.3, seed=72))


def test_bwd_no_state_inputs(cuda_lib):
    check_bwd(cuda_lib, small_cfg("bf16", 128, 64, 90, B=1, H=3, s0=0.0, seed=73), with_dST=False)


def test_bwd_empty_sequence(cuda_lib):
    """T = 0: dS0 = dS_T, nothing else is written."""
    cfg = small_cfg("f32", 64, 64, 0, B=1, H=2, s0=0.3, seed=74)
    x = to_dev(I.prefill_inputs(cfg))
    c = to_dev(I.bwd_cotangents(cfg))
    g = cuda_lib.chunk_bwd(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], x["S0"], c["dO"], c["dST"])
    torch.cuda.synchronize()
    assert torch.equal(g["dS0"], c["dST"])


def test_bwd_deterministic(cuda_lib):
    cfg = small_cfg("bf16", 128, 64, 300, B=2, H=2, s0=0.3, seed=75)
    x = to_dev(I.prefill_inputs(cfg))
    c = to_dev(I.bwd_cotangents(cfg))
    outs = [cuda_lib.chunk_bwd(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], x["S0"], c["dO"], c["dST"])
            for _ in range(2)]
    torch.cuda.synchronize()
    for n in BWD_NAMES:
        assert torch.equal(outs[0][n], outs[1][n]), n


def test_bwd_b4_h32_t8k_sampled(cuda_lib):
    """The B4 H32 T8192 strong-decay workload; two (batch, head) slices against
    the oracle (heads are independent, so the sample is exact)."""
    cfg = I.B4_H32_T8K
    x = to_dev(I.prefill_inputs(cfg))
    c = to_dev(I.bwd_cotangents(cfg))
    g = cuda_lib.chunk_bwd(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], x["S0"], c["dO"], c["dST"])
    torch.cuda.synchronize()
    cc = I.bwd_cotangents(cfg)
    for b, h in [(0, 3), (3, 30)]:
        xs = I.prefill_inputs(cfg, heads=[(b, h)])
        dO = cc["dO"][b:b + 1, :, h:h + 1]
        dST = cc["dST"][b:b + 1, h:h + 1]
        ref = oracle.recurrent_bwd(xs["q"], xs["k"], xs["v"], xs["log_alpha"], xs["beta"], xs["S0"], dO, dST)
        for n in BWD_NAMES:
            got = g[n][b, :, h] if n not in ("dS0",) else g[n][b, h]
            want = ref[n][0, :, 0] if n != "dS0" else ref[n][0, 0]
            e = rel_err(got.float().cpu().numpy(), want)
            print(f"PARITY bwd full b={b} h={h} {n}={e:.2e}")
            assert e <= TOL["bf16"], (b, h, n, e)


@pytest.mark.parametrize("T", [77, 200, 512])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_bwd_low_memory_mode(cuda_lib, dtype, T):
    """One stored state per 64 tokens and the per-block recompute sweep
    (the default for workspaces above 16 GB)."""
    d = 64 if dtype == "f32" else 128
    check_bwd(cuda_lib, small_cfg(dtype, d, 64, T, B=1, H=2, s0=0.3, seed=76), memory="low")


@pytest.mark.parametrize("erase,gate", [(True, "scalar"), (False, "channel")])
def test_bwd_low_memory_variants(cuda_lib, erase, gate):
    check_bwd(cuda_lib, small_cfg("bf16", 128, 64, 150, B=1, H=2, s0=0.3, seed=77), erase, gate, memory="low")


def test_bwd_modes_agree(cuda_lib):
    """Both workspace policies run the same arithmetic: bitwise-equal gradients."""
    cfg = small_cfg("bf16", 128, 64, 300, B=2, H=2, s0=0.3, seed=78)
    x = to_dev(I.prefill_inputs(cfg))
    c = to_dev(I.bwd_cotangents(cfg))
    ga = cuda_lib.chunk_bwd(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], x["S0"], c["dO"], c["dST"], memory="all")
    gl = cuda_lib.chunk_bwd(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], x["S0"], c["dO"], c["dST"], memory="low")
    torch.cuda.synchronize()
    for n in BWD_NAMES:
        assert torch.equal(ga[n], gl[n]), n
