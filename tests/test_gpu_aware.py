"""Attention-aware key basis through the CUDA library vs the fp64 oracle.

NOVA-KV summary, "Methodology > Key Transform Derivation" (Theorem 1): the
key-side transform W_k = M_q^{1/2} E_p is not orthogonal, queries are
projected with W_q = M_q^{-1/2} E_p, and keys are centred by the calibration
mean.  The cache stores c = W_k^T (k - mu), reconstructs k_hat = mu + W_q c,
routes on ||k - k_hat|| / ||k|| and decodes with q~ = W_q^T q and compressed
logits (q . mu + q~ . c) / sqrt(d) (reading R24).  The transform of every kv
head comes from the oracle's Theorem 1 on seeded calibration queries with an
anisotropic covariance and the head's own keys; both sides get the same
bf16-rounded bases and fp32 mean.  Bars as for the plain cache: coefficients
within 1 bf16 ulp plus the fp32 accumulation bound (of |x| and |mu|), routed
sets equal outside 1e-4 of tau, list rows exact, e within 5e-5, decode
||o - o_ref||_inf / ||o_ref||_inf <= 2e-3 -- through the prefill projection,
the small-append kernel, the fused append + decode and both decode kernels.
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


def _aware_bases(K, r_k, seed, Nq=2048):
    """Per kv head: Theorem 1's (W_k, W_q, mu) from calibration queries whose
    covariance decays over a random orthonormal frame, and the head's keys.
    K: [B, T, Hkv, d] float64.  Returns bf16-rounded W_k, W_q [Hkv, d, r_k] and
    the fp32-rounded mean [Hkv, d], all as float64."""
    rng = np.random.default_rng(seed)
    B, T, Hkv, d = K.shape
    Wk = np.zeros((Hkv, d, r_k))
    Wq = np.zeros((Hkv, d, r_k))
    mu = np.zeros((Hkv, d))
    for h in range(Hkv):
        frame = np.linalg.qr(rng.standard_normal((d, d)))[0]
        scales = np.geomspace(3.0, 0.3, d)
        Qc = (rng.standard_normal((Nq, d)) * scales) @ frame.T / np.sqrt(Nq)
        tr = O.key_transform(Qc, K[:, :, h].reshape(-1, d))
        Wk[h], Wq[h] = tr.W_k(r_k), tr.W_q(r_k)
        mu[h] = tr.mu
    bf = lambda a: O.bf16_round(a)
    return bf(Wk), bf(Wq), mu.astype(np.float32).astype(np.float64)


def _setup(w, seed, T_cap=None):
    layer = synth.make_layer(w, 0, seed, device=DEV)
    T_cap = T_cap or synth.pad_to(w.T + 16, 32)
    D = U.dims_of(w, T_cap)
    Wk, Wq, mu = _aware_bases(U.f64(layer["K"]), w.r_k, seed)
    t = lambda a, dt: torch.from_numpy(a).to(dt).to(DEV)
    cache = L.LayerCache(D, t(Wk, torch.bfloat16), layer["U_v"], device=DEV,
                         U_kq=t(Wq, torch.bfloat16), mu_k=t(mu, torch.float32))
    oc = O.Cache.empty(U.oracle_dims(D), Wk, U.f64(layer["U_v"]), U_kq=Wq, mu_k=mu)
    ws = L.make_workspace(D, DEV)
    return layer, D, cache, oc, ws


def _gpu_to_oracle(D, cache, oc):
    gc = U.gpu_to_oracle(D, cache)
    gc.U_kq, gc.mu_k = oc.U_kq, oc.mu_k
    return gc


def _abs_bound(oc, X):
    """sum_i |U_k[i,j]| (|x_i| + |mu_i|): the scale of the fp32 error of U_k^T x - U_k^T mu."""
    return U.coef_abs_bound(oc.U_k, np.abs(X) + np.abs(oc.mu_k)[None, None])


def _compress_both(D, cache, oc, K, V, tau, ws, t_new_b=None, band=None):
    starts = oc.seq_len.copy()
    tb = None if t_new_b is None else torch.tensor(t_new_b, dtype=torch.int32, device=DEV)
    err = U.gpu_compress(D, cache, K, V, tau, ws, t_new_b=tb)
    Kf, Vf = U.f64(K), U.f64(V)
    e_ref, _, _ = O.compress(oc, Kf, Vf, tau, t_new_b=t_new_b)
    torch.cuda.synchronize()
    gc = _gpu_to_oracle(D, cache, oc)
    band = U.check_compress_parity(gc, oc, e_ref, tau, starts, err_gpu=U.f64(err), band=band,
                                   abs_k=_abs_bound(oc, Kf), abs_v=U.coef_abs_bound(oc.U_v, Vf))
    return gc, band


WORKLOADS = [
    ("llama8k_small", synth.workload(1, T=1000, layers=1)),
    ("mha_small", synth.workload(4, T=700, layers=1)),
    ("gqa3", synth.workload(1, Hq=24, T=600, layers=1)),
    ("cuda_cores_32_48", synth.workload(1, r_k=32, r_v=48, T=600, layers=1)),
]


@pytest.mark.parametrize("name,w", WORKLOADS, ids=[n for n, _ in WORKLOADS])
def test_aware_compress_append_and_decode(name, w):
    layer, D, cache, oc, ws = _setup(w, seed=61)
    gc, band = _compress_both(D, cache, oc, layer["K"], layer["V"], w.tau, ws)
    q = layer["q"]
    out = U.f64(U.gpu_decode(D, cache, q, ws))
    assert U.out_rel_err(out, O.decode_attn(gc, U.f64(q))) <= U.OUT_RTOL
    assert U.out_rel_err(out, O.decode_attn(oc, U.f64(q))) <= U.OUT_RTOL
    # decode-time appends through the small-append kernel (3 tokens, then 1)
    Ka, Va = synth.decode_tokens(w, layer["Qk"], layer["Qv"], 6, 61, 0, DEV)
    gc, band = _compress_both(D, cache, oc, Ka[:, :3].contiguous(), Va[:, :3].contiguous(), w.tau, ws,
                              band=band)
    gc, band = _compress_both(D, cache, oc, Ka[:, 3:4].contiguous(), Va[:, 3:4].contiguous(), w.tau, ws,
                              band=band)
    out = U.f64(U.gpu_decode(D, cache, q, ws))
    assert U.out_rel_err(out, O.decode_attn(gc, U.f64(q))) <= U.OUT_RTOL
    # fused append + decode steps
    qs = synth.decode_queries(w, 2, 61, 0, DEV)
    for s in range(2):
        k, v = Ka[:, 4 + s:5 + s].contiguous(), Va[:, 4 + s:5 + s].contiguous()
        starts = oc.seq_len.copy()
        err = torch.full((D.B, D.Hkv, 1), float("nan"), device=DEV)
        o = torch.empty(D.B, D.Hq, D.d, dtype=torch.float32, device=DEV)
        L.lrkv_append_decode_attn(D, cache, k, v, w.tau, qs[s], o, err_out=err, ws=ws)
        kf, vf = U.f64(k), U.f64(v)
        e_ref, _, _ = O.compress(oc, kf, vf, w.tau)
        torch.cuda.synchronize()
        gc = _gpu_to_oracle(D, cache, oc)
        band = U.check_compress_parity(gc, oc, e_ref, w.tau, starts, err_gpu=U.f64(err), band=band,
                                       abs_k=_abs_bound(oc, kf), abs_v=U.coef_abs_bound(oc.U_v, vf))
        assert U.out_rel_err(U.f64(o), O.decode_attn(gc, U.f64(qs[s]))) <= U.OUT_RTOL


def test_aware_decode_on_oracle_written_cache():
    """Decode alone: the oracle writes the attention-aware cache, the GPU reads it."""
    w = synth.workload(1, T=2100, layers=1)
    layer = synth.make_layer(w, 0, 67, device=DEV)
    D = U.dims_of(w, synth.pad_to(w.T, 32))
    Wk, Wq, mu = _aware_bases(U.f64(layer["K"]), w.r_k, 67)
    oc = O.Cache.empty(U.oracle_dims(D), Wk, U.f64(layer["U_v"]), U_kq=Wq, mu_k=mu)
    O.compress(oc, U.f64(layer["K"]), U.f64(layer["V"]), w.tau)
    dims, cache = U.oracle_to_gpu(oc)
    cache.U_kq = torch.from_numpy(Wq).to(torch.bfloat16).to(DEV)
    cache.mu_k = torch.from_numpy(mu).to(torch.float32).to(DEV)
    ws = L.make_workspace(dims, DEV)
    out = U.f64(U.gpu_decode(dims, cache, layer["q"], ws))
    assert U.out_rel_err(out, O.decode_attn(oc, U.f64(layer["q"]))) <= U.OUT_RTOL
    # without the query-side basis and the mean the same cache reads differently
    cache.U_kq, cache.mu_k = None, None
    out2 = U.f64(U.gpu_decode(dims, cache, layer["q"], ws))
    assert U.out_rel_err(out2, O.decode_attn(oc, U.f64(layer["q"]))) > 10 * U.OUT_RTOL
