"""The layer's optional parts on the GPU (ia_prefill_fwd_ex, ia_decode_step_ex)
against the fp64 oracle's extended forward, itself pinned by mpmath brute
force, closed forms and invariants: the RMSNorm with per-head gain and bias on
the SSM input, a step per token (selective writing and memory decay), the
complex readout matrix and the bidirectional layer."""
import numpy as np
import pytest
import torch

import ssm_token_mixer_b200 as ia
from gpu_common import device
from parity import TOL_BF16, TOL_F32, report, slice_rel
from ssm_token_mixer_b200 import synthetic

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dev():
    return device()


def options(B, H, N, dx, dv, M, seed, which):
    g = torch.Generator().manual_seed(seed)
    o = {}
    if "selective" in which:
        o["delta_t"] = torch.exp(np.log(5e-3) + torch.rand(B, H, N, generator=g) * (np.log(2e-1) - np.log(5e-3)))
    if "norm" in which:
        o["gain"] = 0.5 + torch.rand(H, dx + dv, generator=g)
        o["bias"] = 0.3 * torch.randn(H, dx + dv, generator=g)
    if "readout" in which:
        o["W"] = (torch.randn(H, M, M, 2, generator=g) / np.sqrt(M)) + torch.eye(M)[None, :, :, None] * \
            torch.tensor([1.0, 0.0])
    return o


def to_oracle(o):
    r = {k: v for k, v in o.items() if k != "W"}
    if "W" in o:
        W = o["W"].double().numpy()
        r["W"] = W[..., 0] + 1j * W[..., 1]
    return r


CASES = [("selective",), ("norm",), ("readout",), ("selective", "norm", "readout")]


@pytest.mark.parametrize("which", CASES, ids=["+".join(c) for c in CASES])
@pytest.mark.parametrize("dtype,dx,dv,M,tol", [("f32", 16, 12, 8, TOL_F32), ("bf16", 64, 64, 64, TOL_BF16)])
def test_prefill_with_optional_parts(oracle_mod, dev, which, dtype, dx, dv, M, tol):
    B, H, N = 2, 3, 130
    inp = synthetic.layer_inputs(B, H, N, dx, dv, dtype, seed=80 + dx)
    opt = options(B, H, N, dx, dv, M, 81, which)
    delta = None if "selective" in which else inp["delta"]
    g = lambda x: None if x is None else x.to(dev)
    r = ia.prefill_fwd_ex(g(inp["q"]), g(inp["k"]), g(inp["v"]), M, delta=g(delta), want_num_den=True,
                          want_state=True, **{k: g(v) for k, v in opt.items()})
    ia.check_device_errors()
    ref = oracle_mod.forward_ex(inp["q"], inp["k"], inp["v"], M, delta=delta, **to_oracle(opt))
    rep = report(r["num"].cpu(), r["den"].cpu(), r["o"].cpu(), ref)
    assert max(rep.values()) < tol, rep
    st = r["state"].cpu().double().numpy()
    assert np.abs(st - ref["state"]).max() / np.abs(ref["state"]).max() < tol


@pytest.mark.parametrize("dx,dv,M", [(16, 16, 8), (64, 64, 64)], ids=["small", "register_form"])
def test_split_prefill_and_decode_with_optional_parts(oracle_mod, dev, dx, dv, M):
    # P12/P13 with every part on: prefill(N1) -> state -> prefill(N2) and
    # decode steps equal the oracle on the whole sequence (d_xi = d_v = M =
    # 64: the register-resident kernel, also for the in-place decode step)
    B, H, N1, N2, K = 2, 2, 70, 140, 3
    N = N1 + N2 + K
    inp = synthetic.layer_inputs(B, H, N, dx, dv, "f32", seed=82)
    opt = options(B, H, N, dx, dv, M, 83, ("selective", "norm", "readout"))
    ref = oracle_mod.forward_ex(inp["q"], inp["k"], inp["v"], M, **to_oracle(opt))
    g = lambda x: x.to(dev)
    sl = lambda x, a, b: x[:, :, a:b].contiguous()
    kw = lambda a, b: {"delta_t": g(sl(opt["delta_t"], a, b)), "gain": g(opt["gain"]), "bias": g(opt["bias"]),
                       "W": g(opt["W"])}
    r1 = ia.prefill_fwd_ex(*(g(sl(inp[n], 0, N1)) for n in ("q", "k", "v")), M, want_state=True, **kw(0, N1))
    r2 = ia.prefill_fwd_ex(*(g(sl(inp[n], N1, N1 + N2)) for n in ("q", "k", "v")), M, want_state=True,
                           state_in=r1["state"], **kw(N1, N1 + N2))
    o = torch.cat([r1["o"].cpu(), r2["o"].cpu()], dim=2)
    assert slice_rel(o, ref["o"][:, :, :N1 + N2], (-2, -1)) < TOL_F32
    state = r2["state"]
    for t in range(N1 + N2, N):
        tok = lambda n: g(inp[n][:, :, t].contiguous())
        r = ia.decode_step_ex(tok("q"), tok("k"), tok("v"), state, M, delta_t=g(opt["delta_t"][:, :, t].contiguous()),
                              gain=g(opt["gain"]), bias=g(opt["bias"]), W=g(opt["W"]))
        ia.check_device_errors()
        assert slice_rel(r["o"].cpu(), ref["o"][:, :, t], (-1,)) < TOL_F32


@pytest.mark.parametrize("dtype,tol", [("f32", TOL_F32), ("bf16", TOL_BF16)])
def test_bidirectional_layer(oracle_mod, dev, dtype, tol):
    B, H, N, d, M = 2, 3, 90, 16, 8
    inp = synthetic.layer_inputs(B, H, N, d, d, dtype, seed=84)
    opt = options(B, H, N, d, d, M, 85, ("selective",))
    g = lambda x: x.to(dev)
    r = ia.prefill_fwd_ex(g(inp["q"]), g(inp["k"]), g(inp["v"]), M, delta_t=g(opt["delta_t"]), bidirectional=True)
    ia.check_device_errors()
    ref = oracle_mod.forward_bidirectional(inp["q"], inp["k"], inp["v"], M, delta_t=opt["delta_t"])
    assert slice_rel(r["o"].cpu(), ref, (-2, -1)) < tol


def test_no_options_is_the_plain_layer(dev):
    inp = synthetic.layer_inputs(2, 2, 150, 64, 64, "bf16", seed=86)
    g = {k: v.to(dev) for k, v in inp.items()}
    a = ia.prefill_fwd(g["q"], g["k"], g["v"], g["delta"], 64, want_num_den=True)
    b = ia.prefill_fwd_ex(g["q"], g["k"], g["v"], 64, delta=g["delta"], want_num_den=True)
    ia.check_device_errors()
    assert slice_rel(b["num"].cpu(), a["num"].cpu(), (-2, -1)) < TOL_BF16


TC_CASES = [("norm",), ("bidirectional",), ("norm", "bidirectional")]


@pytest.mark.parametrize("which", TC_CASES, ids=["+".join(c) for c in TC_CASES])
@pytest.mark.parametrize("dx,dv,N", [(64, 64, 150), (128, 128, 200), (64, 128, 64), (128, 64, 1)])
def test_tensor_core_optional_parts(oracle_mod, dev, which, dx, dv, N):
    # input stabilisation and the bidirectional layer on the tensor-core chunk
    # pass (a prologue writes the normalised and / or reversed operands; the
    # bidirectional second pass is added back by an epilogue), ragged lengths
    B, H, M = 2, 3, 64
    norm, bidir = "norm" in which, "bidirectional" in which
    assert ia.prefill_ex_path(B, H, N, dx, dv, M, "bf16", norm=norm, bidirectional=bidir) == "tensor_core"
    inp = synthetic.layer_inputs(B, H, N, dx, dv, "bf16", seed=90 + dx + dv + N)
    opt = options(B, H, N, dx, dv, M, 91, which)
    g = lambda x: None if x is None else x.to(dev)
    kw = {k: g(v) for k, v in opt.items()}
    if bidir:
        r = ia.prefill_fwd_ex(g(inp["q"]), g(inp["k"]), g(inp["v"]), M, delta=g(inp["delta"]), bidirectional=True,
                              **kw)
        ia.check_device_errors()
        ref = oracle_mod.forward_bidirectional(inp["q"], inp["k"], inp["v"], M, delta=inp["delta"], **opt)
        assert slice_rel(r["o"].cpu(), ref, (-2, -1)) < TOL_BF16
        return
    r = ia.prefill_fwd_ex(g(inp["q"]), g(inp["k"]), g(inp["v"]), M, delta=g(inp["delta"]), want_num_den=True,
                          want_state=True, **kw)
    ia.check_device_errors()
    ref = oracle_mod.forward_ex(inp["q"], inp["k"], inp["v"], M, delta=inp["delta"], **opt)
    rep = report(r["num"].cpu(), r["den"].cpu(), r["o"].cpu(), ref)
    assert max(rep.values()) < TOL_BF16, rep
    st = r["state"].cpu().double().numpy()
    assert np.abs(st - ref["state"]).max() / np.abs(ref["state"]).max() < TOL_BF16


def test_tensor_core_and_token_serial_optional_parts_agree(dev, monkeypatch):
    # the same call through both forms of ia_prefill_fwd_ex
    B, H, N, d, M = 2, 2, 300, 64, 64
    inp = synthetic.layer_inputs(B, H, N, d, d, "bf16", seed=92)
    opt = options(B, H, N, d, d, M, 93, ("norm",))
    g = {k: v.to(dev) for k, v in inp.items()}
    kw = {k: v.to(dev) for k, v in opt.items()}
    a = ia.prefill_fwd_ex(g["q"], g["k"], g["v"], M, delta=g["delta"], bidirectional=True, **kw)
    monkeypatch.setenv("IA_PREFILL_SIMT", "1")
    assert ia.prefill_ex_path(B, H, N, d, d, M, "bf16", norm=True, bidirectional=True) == "sequential"
    b = ia.prefill_fwd_ex(g["q"], g["k"], g["v"], M, delta=g["delta"], bidirectional=True, **kw)
    ia.check_device_errors()
    assert slice_rel(a["o"].cpu(), b["o"].cpu(), (-2, -1)) < TOL_BF16


def test_optional_parts_paths_and_workspace(dev):
    B, H, N = 2, 3, 150
    tc = lambda **kw: ia.prefill_ex_path(B, H, N, 64, 64, 64, "bf16", **kw)
    assert tc() == "tensor_core"
    assert tc(norm=True) == tc(bidirectional=True) == tc(norm=True, bidirectional=True) == "tensor_core"
    assert tc(readout=True) == tc(norm=True, readout=True) == tc(readout=True, bidirectional=True) == "tensor_core"
    assert tc(selective=True) == tc(selective=True, readout=True) == "sequential"
    assert ia.prefill_ex_path(B, H, N, 128, 128, 64, "bf16", readout=True) == "sequential"   # d_xi = 128
    assert ia.prefill_ex_path(B, H, N, 64, 64, 48, "bf16", norm=True) == "sequential"    # M != 64
    assert ia.prefill_ex_path(B, H, N, 64, 64, 64, "f32", norm=True) == "sequential"     # fp32 inputs
    # a workspace one byte short is refused before anything runs
    inp = synthetic.layer_inputs(B, H, N, 64, 64, "bf16", seed=94)
    g = {k: v.to(dev) for k, v in inp.items()}
    shp = ia.make_shape(B, H, N, 64, 64, 64, "bf16")
    opt = ia.IAOptions()
    opt.bidirectional = 1
    need = ia.load_library().ia_prefill_ex_workspace_bytes(ia.ctypes.byref(shp), ia.ctypes.byref(opt))
    assert need > 0
    ws = torch.empty(need - 1, dtype=torch.uint8, device=dev)
    with pytest.raises(ia.IAError) as err:
        ia.prefill_fwd_ex(g["q"], g["k"], g["v"], 64, delta=g["delta"], bidirectional=True, workspace=ws)
    assert err.value.status == 3   # IA_ERR_WORKSPACE


@pytest.mark.parametrize("dx,dv", [(64, 64), (128, 128)])
def test_tensor_core_stabilised_split_prefill(oracle_mod, dev, dx, dv):
    # P13 on the tensor-core form of the stabilised layer: prefill(N1) ->
    # state -> prefill(N2, state_in) equals the oracle on N1 + N2 (ragged N1)
    B, H, M, N1, N2 = 2, 3, 64, 100, 90
    inp = synthetic.layer_inputs(B, H, N1 + N2, dx, dv, "bf16", seed=95 + dx)
    opt = options(B, H, N1 + N2, dx, dv, M, 96, ("norm",))
    assert ia.prefill_ex_path(B, H, N1, dx, dv, M, "bf16", norm=True) == "tensor_core"
    g = lambda x: x.to(dev)
    sl = lambda x, a, b: x[:, :, a:b].contiguous()
    kw = {k: g(v) for k, v in opt.items()}
    r1 = ia.prefill_fwd_ex(*(g(sl(inp[n], 0, N1)) for n in ("q", "k", "v")), M, delta=g(inp["delta"]),
                           want_state=True, **kw)
    r2 = ia.prefill_fwd_ex(*(g(sl(inp[n], N1, N1 + N2)) for n in ("q", "k", "v")), M, delta=g(inp["delta"]),
                           state_in=r1["state"], want_state=True, **kw)
    ia.check_device_errors()
    ref = oracle_mod.forward_ex(inp["q"], inp["k"], inp["v"], M, delta=inp["delta"], **opt)
    o = torch.cat([r1["o"].cpu(), r2["o"].cpu()], dim=2)
    assert slice_rel(o, ref["o"], (-2, -1)) < TOL_BF16
    st = r2["state"].cpu().double().numpy()
    assert np.abs(st - ref["state"]).max() / np.abs(ref["state"]).max() < TOL_BF16


def mode_params(H, M, seed):
    """Delta [H,M] in the S4D-Lin step range and a general decaying A [2M]."""
    g = torch.Generator().manual_seed(seed)
    delta = torch.exp(np.log(2e-2) + torch.rand(H, M, generator=g) * (np.log(1.2e-1) - np.log(2e-2)))
    A = torch.empty(2 * M)
    A[0::2] = -0.2 - 0.6 * torch.rand(M, generator=g)
    A[1::2] = np.pi * torch.arange(M) + 0.7 * torch.rand(M, generator=g)
    return delta.float(), A.float()


SEG_CASES = [("selective", "norm", "readout"), ("readout",), ("norm",)]


@pytest.mark.parametrize("which", SEG_CASES, ids=["+".join(c) for c in SEG_CASES])
@pytest.mark.parametrize("dx,dv,M", [(16, 12, 8), (64, 64, 64)], ids=["small", "register_form"])
def test_segmented_token_serial_pass(oracle_mod, dev, which, dx, dv, M):
    # The token-serial form cuts 357 tokens into five segments (the last one
    # ragged) around the carry kernel, from the state a 50-token prefix left,
    # with a general A and, without a step per token, a Delta per (head, mode):
    # o and the end state against the oracle on the whole sequence, and o
    # against the single pass that a one-byte workspace leaves.  d_xi = d_v =
    # M = 64 runs the register-resident kernel.
    B, H, P, N = 1, 2, 50, 357
    inp = synthetic.layer_inputs(B, H, P + N, dx, dv, "f32", seed=88)
    opt = options(B, H, P + N, dx, dv, M, 89, which)
    delta, A = mode_params(H, M, 90)
    if "selective" in which:
        delta = None
    ref = oracle_mod.forward_ex(inp["q"], inp["k"], inp["v"], M, delta=delta, A=A, **to_oracle(opt))
    pre = oracle_mod.forward_ex(*(x[:, :, :P] for x in (inp["q"], inp["k"], inp["v"])), M, delta=delta, A=A,
                                **to_oracle({k: (x[:, :, :P] if k == "delta_t" else x) for k, x in opt.items()}))
    g = lambda x: None if x is None else x.to(dev)
    tail = lambda x: g(x[:, :, P:].contiguous())
    kw = {k: (tail(x) if k == "delta_t" else g(x)) for k, x in opt.items()}
    state_in = g(torch.from_numpy(np.asarray(pre["state"], dtype=np.float32).ravel()))
    need = ia.prefill_ex_workspace_bytes(B, H, N, dx, dv, M, "f32", norm="gain" in opt, selective="delta_t" in opt,
                                         readout="W" in opt)
    assert need > 0
    outs = {}
    for name, ws in (("segmented", torch.empty(need, dtype=torch.uint8, device=dev)),
                     ("single", torch.empty(1, dtype=torch.uint8, device=dev))):
        r = ia.prefill_fwd_ex(tail(inp["q"]), tail(inp["k"]), tail(inp["v"]), M, delta=g(delta), A=g(A),
                              state_in=state_in, want_state=True, workspace=ws, **kw)
        ia.check_device_errors()
        outs[name] = r
        assert slice_rel(r["o"].cpu(), ref["o"][:, :, P:], (-2, -1)) < TOL_F32, name
        st = r["state"].cpu().double().numpy()
        want = np.asarray(ref["state"]).ravel()
        assert np.abs(st - want).max() / np.abs(want).max() < TOL_F32, name
    assert slice_rel(outs["segmented"]["o"].cpu(), outs["single"]["o"].cpu().double().numpy(), (-2, -1)) < TOL_F32


def test_segmented_bidirectional_layer(oracle_mod, dev):
    # both directions of the bidirectional layer cut into segments, a step per
    # token (the carry's decay from the summed steps, summed back to front in
    # the second direction)
    B, H, N, d, M = 2, 2, 300, 16, 8
    inp = synthetic.layer_inputs(B, H, N, d, d, "f32", seed=91)
    opt = options(B, H, N, d, d, M, 92, ("selective", "norm"))
    g = lambda x: x.to(dev)
    need = ia.prefill_ex_workspace_bytes(B, H, N, d, d, M, "f32", norm=True, selective=True, bidirectional=True)
    assert need > 0
    r = ia.prefill_fwd_ex(g(inp["q"]), g(inp["k"]), g(inp["v"]), M, bidirectional=True,
                          workspace=torch.empty(need, dtype=torch.uint8, device=dev),
                          **{k: g(v) for k, v in opt.items()})
    ia.check_device_errors()
    ref = oracle_mod.forward_bidirectional(inp["q"], inp["k"], inp["v"], M, **to_oracle(opt))
    assert slice_rel(r["o"].cpu(), ref, (-2, -1)) < TOL_F32


TC_W_CASES = [("readout",), ("norm", "readout"), ("readout", "bidirectional")]


@pytest.mark.parametrize("which", TC_W_CASES, ids=["+".join(c) for c in TC_W_CASES])
@pytest.mark.parametrize("dv", [64, 128])
def test_tensor_core_readout_matrix(oracle_mod, dev, which, dv):
    # the readout matrix on the chunk pass (G_W between the key-state read and
    # the score matrix), d_xi = 64, a ragged N over several chunks, with the
    # stabilisation or the bidirectional layer beside it: o, num, den and the
    # end state against the oracle
    B, H, N, dx, M = 2, 3, 333, 64, 64
    bidir = "bidirectional" in which
    inp = synthetic.layer_inputs(B, H, N, dx, dv, "bf16", seed=97 + dv)
    opt = options(B, H, N, dx, dv, M, 98, which)
    present = dict(norm="gain" in opt, readout=True, bidirectional=bidir)
    assert ia.prefill_ex_path(B, H, N, dx, dv, M, "bf16", **present) == "tensor_core"
    g = lambda x: x.to(dev)
    r = ia.prefill_fwd_ex(g(inp["q"]), g(inp["k"]), g(inp["v"]), M, delta=g(inp["delta"]), bidirectional=bidir,
                          want_num_den=not bidir, want_state=not bidir, **{k: g(v) for k, v in opt.items()})
    ia.check_device_errors()
    if bidir:
        ref = oracle_mod.forward_bidirectional(inp["q"], inp["k"], inp["v"], M, delta=inp["delta"], **to_oracle(opt))
        assert slice_rel(r["o"].cpu(), ref, (-2, -1)) < TOL_BF16
        return
    ref = oracle_mod.forward_ex(inp["q"], inp["k"], inp["v"], M, delta=inp["delta"], **to_oracle(opt))
    rep = report(r["num"].cpu(), r["den"].cpu(), r["o"].cpu(), ref)
    assert max(rep.values()) < TOL_BF16, rep
    st = r["state"].cpu().double().numpy()
    assert np.abs(st - ref["state"]).max() / np.abs(ref["state"]).max() < TOL_BF16


def test_tensor_core_readout_matrix_across_heads_and_ranges(oracle_mod, dev, monkeypatch):
    # forced grids put several heads in one CTA (W' reloaded per head) and
    # start ranges inside streams (look-back; the state-only chain reads no W)
    B, H, N, d, M = 1, 4, 700, 64, 64
    inp = synthetic.layer_inputs(B, H, N, d, d, "bf16", seed=99)
    opt = options(B, H, N, d, d, M, 100, ("readout",))
    ref = oracle_mod.forward_ex(inp["q"], inp["k"], inp["v"], M, delta=inp["delta"], **to_oracle(opt))
    g = lambda x: x.to(dev)
    for grid in ("1", "3", "7"):
        monkeypatch.setenv("IA_PREFILL_GRID", grid)
        r = ia.prefill_fwd_ex(g(inp["q"]), g(inp["k"]), g(inp["v"]), M, delta=g(inp["delta"]), want_num_den=True,
                              W=g(opt["W"]))
        ia.check_device_errors()
        rep = report(r["num"].cpu(), r["den"].cpu(), r["o"].cpu(), ref)
        assert max(rep.values()) < TOL_BF16, (grid, rep)
