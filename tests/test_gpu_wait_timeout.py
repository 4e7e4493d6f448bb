"""Failure handling without a fault: a bounded wait that runs out.

The prefill projection's roles wait on mbarriers with an iteration limit.
With the main-loop limit lowered to one poll (LRKV_MAIN_WAIT_ITERS=1, read by
the library at each prefill-sized lrkv_compress), the MMA issuer gives up on
its first input tile: the call must report LRKV_DEV_WAIT_TIMEOUT in the
cache's status word, return normally (the other roles drain their copies and
MMAs in flight with their full limits, TMEM is freed), and leave the GPU and
the workspace usable: the same workspace then serves a normal call whose
result is oracle-exact.
"""
import pytest
import torch

import oracle as O
import synth
import decode_attention_lrkv_b200 as L
from tests import lrkv_testutil as U

pytestmark = pytest.mark.gpu

DEV = "cuda"


def test_projection_wait_runs_out_then_a_normal_call_is_exact(monkeypatch):
    w = synth.workload(1, T=1500, layers=1)
    layer = synth.make_layer(w, 0, 91, device=DEV)
    D = U.dims_of(w, synth.pad_to(w.T + 8, 32))
    ws = L.make_workspace(D, DEV)
    bad = L.LayerCache(D, layer["U_k"], layer["U_v"], device=DEV)
    monkeypatch.setenv("LRKV_MAIN_WAIT_ITERS", "1")
    L.lrkv_compress(D, bad, layer["K"], layer["V"], w.tau, ws=ws)
    torch.cuda.synchronize()
    assert int(bad.dev_status[0]) & L.DEV_WAIT_TIMEOUT
    monkeypatch.delenv("LRKV_MAIN_WAIT_ITERS")
    # the context and the workspace are still good
    cache = L.LayerCache(D, layer["U_k"], layer["U_v"], device=DEV)
    oc = O.Cache.empty(U.oracle_dims(D), U.f64(layer["U_k"]), U.f64(layer["U_v"]))
    err = U.gpu_compress(D, cache, layer["K"], layer["V"], w.tau, ws)
    Kf, Vf = U.f64(layer["K"]), U.f64(layer["V"])
    e_ref, _, _ = O.compress(oc, Kf, Vf, w.tau)
    torch.cuda.synchronize()
    gc = U.gpu_to_oracle(D, cache)
    assert gc.status == 0
    U.check_compress_parity(gc, oc, e_ref, w.tau, [0], err_gpu=U.f64(err),
                            abs_k=U.coef_abs_bound(oc.U_k, Kf), abs_v=U.coef_abs_bound(oc.U_v, Vf))
    out = U.f64(U.gpu_decode(D, cache, layer["q"], ws))
    assert U.out_rel_err(out, O.decode_attn(gc, U.f64(layer["q"]))) <= U.OUT_RTOL
