"""GPU tests of the library's runtime pieces around the scan kernels:
decoding plans (one argument check, then one launch per token), the control
of the workspace pool, and allocation failure (every call that takes a
workspace returns MAMBA_ERR_OUT_OF_MEMORY without launching a kernel or
writing an output when its allocation fails; the failure is made on the
host by the library's test hook, no device memory is exhausted)."""
import pytest
import torch

import gpu_cases as gc
from selective_state_space_21_b200 import build, scan
from selective_state_space_21_b200.inputs import (make_conv_params, make_cplx_inputs,
                                                  make_dtproj_params, make_inputs)

pytestmark = pytest.mark.gpu

OOM = 4


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    build.build()
    scan.load_library()
    yield
    scan.test_fail_alloc(-1)


def _tokens(x, t):
    return {k: (None if x[k] is None else x[k][:, :, t].contiguous())
            for k in ("u", "delta", "z", "B", "C")}


@pytest.mark.parametrize("conv", [False, True], ids=["plain", "conv"])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16], ids=["f32", "bf16"])
@pytest.mark.parametrize("N", [16, 5])
def test_step_plan_equals_step(conv, dtype, N):
    """A plan run token after token gives bitwise the results of the
    per-call step (same kernel), with and without the convolution prologue."""
    b, d, L = 2, 300, 12
    x = gc.to_device(make_inputs(b, d, L, N, dtype, seed=61 + N, with_dy=False))
    cp = gc.to_device(make_conv_params(d, 4, seed=62)) if conv else None
    slots = {k: torch.empty_like(v) for k, v in _tokens(x, 0).items() if v is not None}
    y_plan = torch.empty(b, d, dtype=dtype, device="cuda")
    st_plan = torch.zeros(b, d, N, device="cuda")
    st_ref = torch.zeros(b, d, N, device="cuda")
    cs_plan = torch.zeros(b, d, 3, device="cuda") if conv else None
    cs_ref = torch.zeros(b, d, 3, device="cuda") if conv else None
    plan = scan.StepPlan(st_plan, slots["u"], slots["delta"], x["delta_bias"], x["A"],
                         slots["B"], slots["C"], x["D"], slots["z"], y_plan,
                         conv_state=cs_plan, conv_w=cp["conv_w"] if conv else None,
                         conv_b=cp["conv_b"] if conv else None)
    launches0 = scan.launch_count()
    for t in range(L):
        tok = _tokens(x, t)
        for k, v in slots.items():
            v.copy_(tok[k])
        plan.run()
        y_ref = torch.empty_like(y_plan)
        if conv:
            scan.mamba_conv_scan_step(st_ref, cs_ref, tok["u"], cp["conv_w"], cp["conv_b"],
                                      tok["delta"], x["delta_bias"], x["A"], tok["B"], tok["C"],
                                      x["D"], tok["z"], y_ref)
        else:
            scan.mamba_scan_step(st_ref, tok["u"], tok["delta"], x["delta_bias"], x["A"],
                                 tok["B"], tok["C"], x["D"], tok["z"], y_ref)
        torch.cuda.synchronize()
        assert torch.equal(y_plan, y_ref), t
    assert scan.launch_count() - launches0 == 2 * L  # one launch per run and per step
    assert torch.equal(st_plan, st_ref)
    if conv:
        assert torch.equal(cs_plan, cs_ref)
    plan.close()
    assert scan.mamba_scan_stream_status() == 0


def test_step_plan_rejects_bad_buffers():
    x = gc.to_device(make_inputs(1, 8, 1, 16, torch.float32, seed=63))
    tok = _tokens(x, 0)
    state = torch.zeros(1, 8, 16, device="cuda")
    y = torch.empty(1, 8, device="cuda")
    with pytest.raises(scan.MambaScanError):  # y overlaps an input
        scan.StepPlan(state, tok["u"], tok["delta"], x["delta_bias"], x["A"], tok["B"],
                      tok["C"], x["D"], tok["z"], tok["u"])
    lib = scan.load_library()
    import ctypes
    h = ctypes.c_void_p()
    # conv_state given without a convolution width
    rc = lib.mamba_scan_step_plan_create(ctypes.byref(h), state.data_ptr(), state.data_ptr(),
                                         tok["u"].data_ptr(), None, None, 0,
                                         tok["delta"].data_ptr(), None, x["A"].data_ptr(),
                                         tok["B"].data_ptr(), tok["C"].data_ptr(), None, None,
                                         y.data_ptr(), 1, 8, 16, 0)
    assert rc == 1 and not h.value
    assert lib.mamba_scan_step_plan_run(None, None) == 1
    lib.mamba_scan_step_plan_destroy(None)


def test_pool_reserve_trim_and_report():
    """The pool holds the workspace of a backward after it finishes (its
    reserve keeps it mapped); a trim to 0 gives it back."""
    x = gc.to_device(make_inputs(2, 256, 1024, 16, torch.bfloat16, seed=64, with_dy=True))
    gc.gpu_bwd(x)
    torch.cuda.synchronize()
    held = scan.pool_reserved()
    assert held > 0
    scan.pool_trim(0)
    torch.cuda.synchronize()
    assert scan.pool_reserved() == 0
    try:
        scan.pool_set_reserve(0)
        gc.gpu_bwd(x)
        torch.cuda.synchronize()
        assert scan.pool_reserved() == 0  # given back at the synchronization
    finally:
        scan.pool_set_reserve(4 << 30)
    g1 = gc.gpu_bwd(x)
    g2 = gc.gpu_bwd(x)
    for k in g1:
        assert torch.equal(g1[k], g2[k]), k
    assert scan.pool_reserved() > 0


def _nan_like(t):
    return torch.full_like(t, float("nan"))


def _calls():
    """(name, inputs, function(outputs) -> None, output makers) for every
    entry point that takes a workspace."""
    out = []
    f = gc.to_device(make_inputs(2, 200, 512, 16, torch.bfloat16, seed=65, with_dy=True))
    r = gc.to_device(make_inputs(2, 70, 50, 16, torch.float32, seed=66, with_dy=True))
    cp = gc.to_device(make_conv_params(200, 4, seed=67))
    cx = gc.to_device(make_cplx_inputs(2, 70, 64, 8, torch.float32, seed=68, with_dy=True))
    pp = gc.to_device(make_dtproj_params(2, 200, 512, 8, torch.bfloat16, seed=69))
    f32 = dict(device="cuda", dtype=torch.float32)

    def fwd_outs(x):
        return {"y": _nan_like(x["u"]), "last": torch.full((x["u"].shape[0], x["u"].shape[1],
                                                            x["A"].shape[1]), float("nan"),
                                                           device="cuda")}

    def bwd_outs(x):
        d, n = x["A"].shape
        return {"du": _nan_like(x["u"]), "dd": _nan_like(x["u"]), "dz": _nan_like(x["u"]),
                "dB": _nan_like(x["B"]), "dC": _nan_like(x["C"]),
                "dA": torch.full((d, n), float("nan"), **f32),
                "dD": torch.full((d,), float("nan"), **f32),
                "db": torch.full((d,), float("nan"), **f32)}

    out.append(("fwd staged", lambda o: scan.mamba_scan_fwd(
        f["u"], f["delta"], f["delta_bias"], f["A"], f["B"], f["C"], f["D"], f["z"], o["y"],
        o["last"]), lambda: fwd_outs(f)))
    out.append(("fwd three-phase", lambda o: scan.mamba_scan_fwd(
        f["u"], f["delta"], f["delta_bias"], f["A"], f["B"], f["C"], f["D"], f["z"], o["y"],
        o["last"], chunk_len=128, carry="three_phase"), lambda: fwd_outs(f)))
    for name, x in (("bwd staged", f), ("bwd reference", r)):
        out.append((name, lambda o, x=x: scan.mamba_scan_bwd(
            x["u"], x["delta"], x["delta_bias"], x["A"], x["B"], x["C"], x["D"], x["z"], x["dy"],
            o["du"], o["dd"], o["dA"], o["dB"], o["dC"], o["dD"], o["dz"], o["db"]),
            lambda x=x: bwd_outs(x)))
    out.append(("bwd three-phase", lambda o: scan.mamba_scan_bwd(
        f["u"], f["delta"], f["delta_bias"], f["A"], f["B"], f["C"], f["D"], f["z"], f["dy"],
        o["du"], o["dd"], o["dA"], o["dB"], o["dC"], o["dD"], o["dz"], o["db"], chunk_len=128,
        carry="three_phase"), lambda: bwd_outs(f)))

    def conv_outs():
        o = bwd_outs(f)
        o["dcw"] = torch.full((200, 4), float("nan"), **f32)
        o["dcb"] = torch.full((200,), float("nan"), **f32)
        return o

    out.append(("conv fwd", lambda o: scan.mamba_conv_scan_fwd(
        f["u"], cp["conv_w"], cp["conv_b"], f["delta"], f["delta_bias"], f["A"], f["B"], f["C"],
        f["D"], f["z"], o["y"], o["last"]), lambda: fwd_outs(f)))
    out.append(("conv bwd", lambda o: scan.mamba_conv_scan_bwd(
        f["u"], cp["conv_w"], cp["conv_b"], f["delta"], f["delta_bias"], f["A"], f["B"], f["C"],
        f["D"], f["z"], f["dy"], o["du"], o["dcw"], o["dcb"], o["dd"], o["dA"], o["dB"], o["dC"],
        o["dD"], o["dz"], o["db"]), conv_outs))
    out.append(("cplx bwd", lambda o: scan.mamba_cplx_scan_bwd(
        cx["u"], cx["delta"], cx["delta_bias"], cx["A"], cx["B"], cx["C"], cx["D"], cx["z"],
        cx["dy"], o["du"], o["dd"], o["dA"], o["dB"], o["dC"], o["dD"], o["dz"], o["db"]),
        lambda: bwd_outs(cx)))

    def dtp_outs():
        o = bwd_outs(f)
        del o["dd"]  # the projection's backward returns d_dt_low and dW_dt in its place
        o["ddl"] = _nan_like(pp["dt_low"])
        o["dW"] = torch.full((200, 8), float("nan"), **f32)
        return o

    out.append(("dtproj fwd", lambda o: scan.mamba_dtproj_scan_fwd(
        f["u"], pp["dt_low"], pp["W_dt"], f["delta_bias"], f["A"], f["B"], f["C"], f["D"], f["z"],
        o["y"], o["last"]), lambda: fwd_outs(f)))
    out.append(("dtproj bwd", lambda o: scan.mamba_dtproj_scan_bwd(
        f["u"], pp["dt_low"], pp["W_dt"], f["delta_bias"], f["A"], f["B"], f["C"], f["D"], f["z"],
        f["dy"], o["du"], o["ddl"], o["dW"], o["dA"], o["dB"], o["dC"], o["dD"], o["dz"], o["db"]),
        dtp_outs))

    # the training pairs: the backward reads a buffer its forward filled
    saved = torch.empty(scan.saved_bytes(2, 200, 512, 16, torch.bfloat16), device="cuda",
                        dtype=torch.uint8)
    csaved = torch.empty(scan.conv_saved_bytes(2, 200, 512, 16, 4, torch.bfloat16),
                         device="cuda", dtype=torch.uint8)
    scan.mamba_scan_fwd_save(f["u"], f["delta"], f["delta_bias"], f["A"], f["B"], f["C"], f["D"],
                             f["z"], torch.empty_like(f["u"]), None, saved)
    scan.mamba_conv_scan_fwd_save(f["u"], cp["conv_w"], cp["conv_b"], f["delta"], f["delta_bias"],
                                  f["A"], f["B"], f["C"], f["D"], f["z"], torch.empty_like(f["u"]),
                                  None, csaved)
    torch.cuda.synchronize()
    out.append(("fwd save", lambda o: scan.mamba_scan_fwd_save(
        f["u"], f["delta"], f["delta_bias"], f["A"], f["B"], f["C"], f["D"], f["z"], o["y"],
        o["last"], torch.empty_like(saved)), lambda: fwd_outs(f)))
    out.append(("bwd saved", lambda o: scan.mamba_scan_bwd_saved(
        f["u"], f["delta"], f["delta_bias"], f["A"], f["B"], f["C"], f["D"], f["z"], f["dy"],
        o["du"], o["dd"], o["dA"], o["dB"], o["dC"], o["dD"], o["dz"], o["db"], saved),
        lambda: bwd_outs(f)))
    out.append(("conv fwd save", lambda o: scan.mamba_conv_scan_fwd_save(
        f["u"], cp["conv_w"], cp["conv_b"], f["delta"], f["delta_bias"], f["A"], f["B"], f["C"],
        f["D"], f["z"], o["y"], o["last"], torch.empty_like(csaved)), lambda: fwd_outs(f)))
    out.append(("conv bwd saved", lambda o: scan.mamba_conv_scan_bwd_saved(
        f["u"], cp["conv_w"], cp["conv_b"], f["delta"], f["delta_bias"], f["A"], f["B"], f["C"],
        f["D"], f["z"], f["dy"], o["du"], o["dcw"], o["dcb"], o["dd"], o["dA"], o["dB"], o["dC"],
        o["dD"], o["dz"], o["db"], csaved), conv_outs))
    xsaved = torch.empty(scan.cplx_saved_bytes(2, 70, 64, 8, torch.float32), device="cuda",
                         dtype=torch.uint8)
    scan.mamba_cplx_scan_fwd_save(cx["u"], cx["delta"], cx["delta_bias"], cx["A"], cx["B"], cx["C"],
                                  cx["D"], cx["z"], torch.empty_like(cx["u"]), None, xsaved)
    torch.cuda.synchronize()
    out.append(("cplx bwd saved", lambda o: scan.mamba_cplx_scan_bwd_saved(
        cx["u"], cx["delta"], cx["delta_bias"], cx["A"], cx["B"], cx["C"], cx["D"], cx["z"],
        cx["dy"], o["du"], o["dd"], o["dA"], o["dB"], o["dC"], o["dD"], o["dz"], o["db"], xsaved),
        lambda: bwd_outs(cx)))
    # the projection's pair stores states where its backward runs in one
    # chunk (L <= 256)
    fs = gc.to_device(make_inputs(2, 200, 256, 16, torch.bfloat16, seed=70, with_dy=True))
    ps = gc.to_device(make_dtproj_params(2, 200, 256, 8, torch.bfloat16, seed=71))
    psaved = torch.empty(scan.dtproj_saved_bytes(2, 200, 256, 16, 8, torch.bfloat16),
                         device="cuda", dtype=torch.uint8)
    assert psaved.numel() > 0
    scan.mamba_dtproj_scan_fwd_save(fs["u"], ps["dt_low"], ps["W_dt"], fs["delta_bias"], fs["A"],
                                    fs["B"], fs["C"], fs["D"], fs["z"], torch.empty_like(fs["u"]),
                                    None, psaved)
    torch.cuda.synchronize()

    def dtps_outs():
        o = bwd_outs(fs)
        del o["dd"]
        o["ddl"] = _nan_like(ps["dt_low"])
        o["dW"] = torch.full((200, 8), float("nan"), **f32)
        return o

    out.append(("dtproj fwd save", lambda o: scan.mamba_dtproj_scan_fwd_save(
        fs["u"], ps["dt_low"], ps["W_dt"], fs["delta_bias"], fs["A"], fs["B"], fs["C"], fs["D"],
        fs["z"], o["y"], o["last"], torch.empty_like(psaved)), lambda: fwd_outs(fs)))
    out.append(("dtproj bwd saved", lambda o: scan.mamba_dtproj_scan_bwd_saved(
        fs["u"], ps["dt_low"], ps["W_dt"], fs["delta_bias"], fs["A"], fs["B"], fs["C"], fs["D"],
        fs["z"], fs["dy"], o["du"], o["ddl"], o["dW"], o["dA"], o["dB"], o["dC"], o["dD"],
        o["dz"], o["db"], psaved), dtps_outs))
    return out


@pytest.mark.parametrize("index", range(17))
def test_allocation_failure_returns_oom_and_launches_nothing(index):
    calls = _calls()
    name, fn, make_out = calls[index]
    saw_oom = False
    for after in range(4):
        o = make_out()
        torch.cuda.synchronize()
        launches0 = scan.launch_count()
        scan.test_fail_alloc(after)
        try:
            fn(o)
            status = 0
        except scan.MambaScanError as e:
            status = e.status
        finally:
            scan.test_fail_alloc(-1)
        torch.cuda.synchronize()
        if status == OOM:
            saw_oom = True
            assert scan.launch_count() == launches0, f"{name}: a kernel ran after the failure"
            for k, v in o.items():
                assert torch.isnan(v.float()).all(), f"{name}: {k} was written"
        else:
            assert status == 0, f"{name}: status {status}"
            assert scan.launch_count() > launches0
    assert saw_oom, name
    assert scan.mamba_scan_stream_status() == 0
    o = make_out()
    fn(o)
    torch.cuda.synchronize()
    for k, v in o.items():
        assert torch.isfinite(v.float()).all(), f"{name}: {k} after a normal call"
