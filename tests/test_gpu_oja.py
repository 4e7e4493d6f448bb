"""lrkv_oja_update (OjaKV's online basis update, reading R23) vs the fp64 oracle.

OjaKV repository README, "Method Summary > OjaKV": the subspace follows the
context with Oja's algorithm during prefill (a batch step over a chunk of rows)
and decoding (one step per new row).  The GPU sums in fp32 and steps and
re-orthonormalises in fp64; the oracle (oracle/oja.py) is fp64 throughout and
takes the same fp32 starting basis and bf16 rows.  Bars: the fp32 basis within
2e-5 of the oracle's per entry, orthonormal columns to 1e-5, and the bf16
rounding within half a bf16 ulp (+ the same 2e-5) of the oracle's basis.
"""
import numpy as np
import pytest
import torch

import oracle as O
import synth
import decode_attention_lrkv_b200 as L
from tests import lrkv_testutil as U

pytestmark = pytest.mark.gpu

DEV = "cuda"
ATOL = 2e-5


def _check(U_gpu, U_bf, U_ref):
    U_gpu = U_gpu.double().cpu().numpy()
    assert np.abs(U_gpu - U_ref).max() <= ATOL
    for h in range(U_gpu.shape[0]):
        G = U_gpu[h].T @ U_gpu[h]
        assert np.abs(G - np.eye(G.shape[0])).max() <= 1e-5
    if U_bf is not None:
        ub = U.f64(U_bf)
        assert np.all(np.abs(ub - U_ref) <= O.bf16_ulp(np.abs(U_ref)) / 2 + ATOL)


@pytest.mark.parametrize("wi,r,n_rows,eta", [(1, 64, 3000, 0.1), (2, 48, 777, 0.5), (4, 64, 129, 0.05),
                                             (1, 96, 64, 1.0), (1, 128, 200, 0.2), (0, 16, 512, 0.3)])
def test_batch_step_matches_oracle(wi, r, n_rows, eta):
    w = synth.workload(wi, T=n_rows, layers=1)
    layer = synth.make_layer(w, 0, 81, device=DEV)
    D = L.Dims(B=w.B, Hq=w.Hq, Hkv=w.Hkv, d=w.d, r_k=w.r_k, r_v=w.r_v, T_cap=32, F_cap=0)
    U0 = layer["Qk"][:, :, :r].contiguous()                  # fp32, orthonormal columns
    Ug = U0.clone()
    U_bf = torch.empty(w.Hkv, w.d, r, dtype=torch.bfloat16, device=DEV)
    X = layer["K"]                                            # [B, T, Hkv, d] bf16
    L.lrkv_oja_update(D, X, Ug, eta, U_out=U_bf)
    torch.cuda.synchronize()
    Xf = U.f64(X).reshape(-1, w.Hkv, w.d)
    U0f = U0.double().cpu().numpy()
    ref = np.stack([O.oja_step(U0f[h], Xf[:, h], eta) for h in range(w.Hkv)])
    _check(Ug, U_bf, ref)


def test_decode_steps_match_oracle_stream():
    """One step per new row (decode), eight in a row, each from the last."""
    w = synth.workload(1, T=8, layers=1)
    layer = synth.make_layer(w, 0, 83, device=DEV)
    D = L.Dims(B=1, Hq=w.Hq, Hkv=w.Hkv, d=w.d, r_k=w.r_k, r_v=w.r_v, T_cap=32, F_cap=0)
    U0 = layer["Qv"][:, :, :w.r_v].contiguous()
    Ug = U0.clone()
    X = layer["V"]                                            # [1, 8, Hkv, d]
    for t in range(8):
        L.lrkv_oja_update(D, X[:, t:t + 1].contiguous(), Ug, 0.2)
    torch.cuda.synchronize()
    Xf = U.f64(X)[0]
    U0f = U0.double().cpu().numpy()
    ref = np.stack([O.oja_stream(U0f[h], Xf[:, h], 0.2) for h in range(w.Hkv)])
    _check(Ug, None, ref)


def test_zero_step_keeps_the_basis():
    """eta = 0 leaves an orthonormal basis where it is (up to the fp32 storage)."""
    w = synth.workload(4, T=300, layers=1)
    layer = synth.make_layer(w, 0, 85, device=DEV)
    D = L.Dims(B=1, Hq=w.Hq, Hkv=w.Hkv, d=w.d, r_k=w.r_k, r_v=w.r_v, T_cap=32, F_cap=0)
    U0 = layer["Qk"][:, :, :48].contiguous()
    Ug = U0.clone()
    L.lrkv_oja_update(D, layer["K"], Ug, 0.0)
    torch.cuda.synchronize()
    assert (Ug - U0).abs().max().item() <= 1e-6


def test_update_then_decode_reads_the_new_basis():
    """An update that writes a cache's value basis in place (U_out = the
    cache's U_v), then a decode issued right after it on the same stream: the
    decode (which loads the bases before waiting on the preceding kernel)
    attends with the updated basis.  Checked against the oracle's decode over
    the same cache contents with that basis."""
    w = synth.workload(1, T=700, layers=1)
    layer = synth.make_layer(w, 0, 87, device=DEV)
    D = U.dims_of(w, synth.pad_to(w.T, 32))
    cache = L.LayerCache(D, layer["U_k"], layer["U_v"].clone(), device=DEV)
    ws = L.make_workspace(D, DEV)
    L.lrkv_compress(D, cache, layer["K"], layer["V"], w.tau, ws=ws)
    Uf = layer["Qv"][:, :, :w.r_v].contiguous()          # fp32 orthonormal start
    X = layer["V"][0, :256].contiguous()                  # [256, Hkv, d]
    torch.cuda.synchronize()
    L.lrkv_oja_update(D, X.unsqueeze(0), Uf, 0.5, U_out=cache.U_v)
    out = U.f64(U.gpu_decode(D, cache, layer["q"], ws))
    torch.cuda.synchronize()
    gc = U.gpu_to_oracle(D, cache)                        # holds the updated U_v
    assert U.out_rel_err(out, O.decode_attn(gc, U.f64(layer["q"]))) <= U.OUT_RTOL
    # the basis did change
    assert (cache.U_v.float() - layer["U_v"].float()).abs().max().item() > 1e-3
