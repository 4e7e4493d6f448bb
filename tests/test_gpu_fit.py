"""lrkv_fit_basis (StaticPCA's offline basis on the GPU) vs the fp64 oracle.

Bars, per kv head: every eigenvalue within 1e-5 of the largest one; the
rank-r span at least as good as the oracle's to 1e-3 relative in the
residual sum of squares (Eckart-Young: the oracle's residual is the
discarded eigenvalue mass, the minimum over all rank-r subspaces); columns
whose eigenvalue is separated from its neighbours by more than 1% equal the
oracle's bf16-rounded, sign-fixed eigenvectors within 2e-3; exact low-rank
data gives exactly its basis.
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


def _check_head(Xh, Ug, lam_g, r):
    """Xh [N, d] fp64 rows; Ug [d, r] fp64 (the GPU's bf16 basis); lam_g [d] descending."""
    Ur, lam = O.fit_basis(Xh, r)
    assert np.abs(lam_g - lam).max() <= 1e-5 * lam[0]
    Q, _ = np.linalg.qr(Ug)                       # the span of the GPU's columns
    resid = ((Xh - Xh @ Q @ Q.T) ** 2).sum()
    opt = lam[r:].sum()
    assert resid <= opt + 1e-3 * max(opt, 1e-12 * lam[0]) + 1e-9 * lam[0], (resid, opt)
    gap = np.full(r, np.inf)
    for k in range(r):
        for j in (k - 1, k + 1):
            if 0 <= j < len(lam):
                gap[k] = min(gap[k], abs(lam[k] - lam[j]) / lam[0])
    for k in np.flatnonzero(gap > 1e-2):
        assert np.abs(Ug[:, k] - O.bf16_round(Ur[:, k])).max() <= 2e-3, k


@pytest.mark.parametrize("wi,T,r", [(1, 2048, 64), (2, 3000, 48), (4, 777, 48), (0, 512, 32)])
def test_fit_basis_matches_oracle(wi, T, r):
    w = synth.workload(wi, T=T, layers=1)
    layer = synth.make_layer(w, 0, 51, device=DEV)
    D = U.dims_of(w, synth.pad_to(T, 32))
    heads = range(min(w.Hkv, 4))
    for X in (layer["K"], layer["V"]):
        Ug, lam_g = L.lrkv_fit_basis(D, X, r)
        torch.cuda.synchronize()
        Xf = U.f64(X)
        for h in heads:
            _check_head(Xf[:, :, h].reshape(-1, w.d), U.f64(Ug[h]), U.f64(lam_g[h]), r)


def test_fit_basis_exact_low_rank_rows():
    """Each row a multiple of one of r unit vectors (G diagonal, distinct masses): the basis
    is exactly those vectors, ordered by mass, and the rest of the spectrum is 0."""
    d, Hkv, r, N = 128, 2, 8, 320
    g = torch.Generator().manual_seed(5)
    idx = torch.randperm(d, generator=g)[:r]
    scale = torch.linspace(3.0, 1.0, r)
    X = torch.zeros(N, Hkv, d)
    for n in range(N):
        X[n, :, idx[n % r]] = torch.randn(Hkv, generator=g) * scale[n % r]
    X = X.to(torch.bfloat16).to(DEV)
    D = L.Dims(B=1, Hq=Hkv, Hkv=Hkv, d=d, r_k=16, r_v=16, T_cap=320, F_cap=0)
    Ug, lam_g = L.lrkv_fit_basis(D, X, r)
    torch.cuda.synchronize()
    Xf = U.f64(X)
    for h in range(Hkv):
        Ur, lam = O.fit_basis(Xf[:, h], r)
        assert np.array_equal(U.f64(Ug[h]), O.bf16_round(Ur))
        assert np.abs(U.f64(lam_g[h])[r:]).max() <= 1e-6 * lam[0]


@pytest.mark.parametrize("N", [1, 5, 63, 64, 65, 200])
def test_fit_basis_few_rows(N):
    w = synth.workload(1, T=max(N, 1), layers=1)
    layer = synth.make_layer(w, 0, 53, device=DEV)
    X = layer["K"][:, :N, :2].contiguous()
    D = L.Dims(B=1, Hq=8, Hkv=2, d=128, r_k=16, r_v=16, T_cap=256, F_cap=0)
    r = min(16, N)
    Ug, lam_g = L.lrkv_fit_basis(D, X, r)
    torch.cuda.synchronize()
    Xf = U.f64(X)
    for h in range(2):
        Xh = Xf[0, :, h]
        _, lam = O.fit_basis(Xh, r)
        assert np.abs(U.f64(lam_g[h]) - lam).max() <= 1e-5 * lam[0]
        Q, _ = np.linalg.qr(U.f64(Ug[h]))
        resid = ((Xh - Xh @ Q @ Q.T) ** 2).sum()
        assert resid <= lam[r:].sum() + 1e-3 * lam[0]


def test_fitted_basis_feeds_compress_and_decode():
    """A basis fitted on the GPU from calibration rows, then the whole path on fresh rows."""
    w = synth.workload(1, T=1200, layers=1)
    calib = synth.make_layer(w, 0, 57, device=DEV)
    layer = synth.make_layer(w, 0, 59, device=DEV)
    D = U.dims_of(w, synth.pad_to(w.T + 4, 32))
    Uk, _ = L.lrkv_fit_basis(D, calib["K"], w.r_k)
    Uv, _ = L.lrkv_fit_basis(D, calib["V"], w.r_v)
    cache = L.LayerCache(D, Uk, Uv, device=DEV)
    oc = O.Cache.empty(U.oracle_dims(D), U.f64(Uk), U.f64(Uv))
    ws = L.make_workspace(D, DEV)
    err = U.gpu_compress(D, cache, layer["K"], layer["V"], w.tau, ws)
    e_ref, _, _ = O.compress(oc, U.f64(layer["K"]), U.f64(layer["V"]), w.tau)
    torch.cuda.synchronize()
    gc = U.gpu_to_oracle(D, cache)
    U.check_compress_parity(gc, oc, e_ref, w.tau, np.zeros(D.B, np.int64), err_gpu=U.f64(err),
                            abs_k=U.coef_abs_bound(oc.U_k, U.f64(layer["K"])),
                            abs_v=U.coef_abs_bound(oc.U_v, U.f64(layer["V"])))
    out = U.f64(U.gpu_decode(D, cache, layer["q"], ws))
    assert U.out_rel_err(out, O.decode_attn(gc, U.f64(layer["q"]))) <= U.OUT_RTOL


@pytest.mark.parametrize("budget", [0.3, 0.1, 0.03])
def test_rank_for_budget_on_fitted_spectra(budget):
    """Rank by error budget from the GPU's eigenvalues: the oracle's rank on its own fp64
    spectrum (or a neighbour, only where the discarded mass is within the eigenvalue
    tolerance of the limit), and the chosen columns' residual within the budget."""
    w = synth.workload(1, T=2048, layers=1)
    layer = synth.make_layer(w, 0, 61, device=DEV)
    D = U.dims_of(w, synth.pad_to(2048, 32))
    Ug, lam_g = L.lrkv_fit_basis(D, layer["K"], 128)
    torch.cuda.synchronize()
    r_g = L.lrkv_rank_for_budget(lam_g, budget).tolist()
    Xf = U.f64(layer["K"])
    for h in range(min(w.Hkv, 4)):
        Xh = Xf[:, :, h].reshape(-1, w.d)
        _, lam = O.fit_basis(Xh, 1)
        lp = np.where(lam > 0, lam, 0.0)
        tot = lp.sum()
        r_o = O.rank_for_budget(lam, budget)
        if r_g[h] != r_o:
            r = min(r_g[h], r_o)
            assert abs(max(r_g[h], r_o) - r) == 1
            assert abs(lp[r:].sum() - budget * tot) <= 2e-3 * lam[0], (h, r_g[h], r_o)
        Q, _ = np.linalg.qr(U.f64(Ug[h])[:, :r_g[h]])
        resid = ((Xh - Xh @ Q @ Q.T) ** 2).sum()
        assert resid <= budget * tot + 2e-3 * lam[0], (h, resid / tot)
