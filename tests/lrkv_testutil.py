"""Helpers shared by the GPU parity tests: move caches between the CUDA
library's torch buffers and the oracle's numpy arrays, and compare them."""
import numpy as np
import torch

import oracle as O
import decode_attention_lrkv_b200 as L

BAND = 1e-4          # routed sets may differ only for tokens with |e - tau| < BAND
OUT_RTOL = 2e-3      # ||o - o_ref||_inf / ||o_ref||_inf per decode call (fp32 out from bf16 in)
ERR_ATOL = 5e-5      # |e_gpu - e_ref| (fp32 vs fp64 error of the error itself)
# Coefficients: the GPU accumulates c = sum_i U_ij x_i (128 products, each exact in fp32)
# in fp32, the oracle in fp64; both then round to bf16.  |RNE(a) - RNE(b)| <= |a - b| +
# ulp, and the fp32 sum is off by at most gamma_n * sum_i |U_ij x_i| with
# gamma_n = n u / (1 - n u), u = 2^-24 (the textbook dot-product bound).  A factor 2
# covers tensor-core accumulation, whose internal rounding order is not sequential.
GAMMA_128 = 128 * 2.0 ** -24 / (1 - 128 * 2.0 ** -24)
COEF_ABS_SAFETY = 2.0


def coef_abs_bound(U, X):
    """sum_i |U[h,i,j]| |x[b,t,h,i]| -> [B, Hkv, t, r]: scale of the fp32 accumulation error."""
    return np.einsum("bthi,hij->bhtj", np.abs(X), np.abs(U))


def f64(t):
    return t.detach().float().cpu().double().numpy()


def dims_of(w, T_cap, F_cap=None, B=None, coef_bits=0):
    return L.Dims(B=B or w.B, Hq=w.Hq, Hkv=w.Hkv, d=w.d, r_k=w.r_k, r_v=w.r_v, T_cap=T_cap,
                  F_cap=T_cap if F_cap is None else F_cap, coef_bits=coef_bits)


def oracle_dims(D):
    return O.Dims(B=D.B, Hq=D.Hq, Hkv=D.Hkv, d=D.d, r_k=D.r_k, r_v=D.r_v, T_cap=D.T_cap,
                  F_cap=D.F_cap)


def gpu_to_oracle(D, cache):
    """An oracle Cache holding exactly the GPU cache's contents."""
    c = O.Cache.empty(oracle_dims(D), f64(cache.U_k), f64(cache.U_v))
    c.coef_k[:] = f64(cache.coef_k)
    c.coef_v[:] = f64(cache.coef_v)
    c.route_mask[:] = cache.route_mask.cpu().numpy().view(np.uint32)
    if D.F_cap:
        c.full_idx[:] = cache.full_idx.cpu().numpy()[:, :, :D.F_cap]
        c.full_k[:] = f64(cache.full_k)[:, :, :D.F_cap]
        c.full_v[:] = f64(cache.full_v)[:, :, :D.F_cap]
    c.full_cnt[:] = cache.full_cnt.cpu().numpy()
    c.seq_len[:] = cache.seq_len.cpu().numpy()
    c.status = int(cache.dev_status[0].item()) & 0xFFFFFFFF
    return c


def oracle_to_gpu(oc, device="cuda"):
    """A LayerCache on the GPU holding exactly the oracle cache's contents."""
    D = oc.dims
    dims = L.Dims(B=D.B, Hq=D.Hq, Hkv=D.Hkv, d=D.d, r_k=D.r_k, r_v=D.r_v, T_cap=D.T_cap,
                  F_cap=D.F_cap)
    bf = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(torch.bfloat16).to(device)
    cache = L.LayerCache(dims, bf(oc.U_k), bf(oc.U_v), device=device)
    cache.coef_k.copy_(bf(oc.coef_k))
    cache.coef_v.copy_(bf(oc.coef_v))
    cache.route_mask.copy_(torch.from_numpy(oc.route_mask.view(np.int32)).to(device))
    if D.F_cap:
        cache.full_idx[:, :, :D.F_cap].copy_(torch.from_numpy(oc.full_idx).to(device))
        cache.full_k[:, :, :D.F_cap].copy_(bf(oc.full_k))
        cache.full_v[:, :, :D.F_cap].copy_(bf(oc.full_v))
    cache.full_cnt.copy_(torch.from_numpy(oc.full_cnt).to(device))
    cache.seq_len.copy_(torch.from_numpy(oc.seq_len).to(device))
    return dims, cache


def gpu_compress(dims, cache, K, V, tau, ws, t_new_b=None, with_err=True):
    """Run lrkv_compress; returns err_out [B,Hkv,t_new] (NaN-filled where unwritten)."""
    err = None
    if with_err:
        err = torch.full((dims.B, dims.Hkv, K.shape[1]), float("nan"), device=K.device)
    L.lrkv_compress(dims, cache, K, V, tau, t_new_b=t_new_b, err_out=err, ws=ws)
    return err


def gpu_decode(dims, cache, q, ws):
    out = torch.empty(dims.B, dims.Hq, dims.d, dtype=torch.float32, device=q.device)
    L.lrkv_decode_attn(dims, cache, q, out, ws=ws)
    return out


def out_rel_err(o, ref):
    o = np.asarray(o, np.float64)
    ref = np.asarray(ref, np.float64)
    den = np.abs(ref).max()
    return np.abs(o - ref).max() / (den if den > 0 else 1.0)


def routed_positions(c, b, h):
    T = int(c.seq_len[b])
    return np.flatnonzero(c.routed(b, h, np.arange(T))) if T else np.zeros(0, np.int64)


def check_compress_parity(gc, oc, e_ref, tau, starts, err_gpu=None, rows=None, band=None,
                          abs_k=None, abs_v=None):
    """Element-by-element comparison of a GPU-written cache with the oracle's.

    e_ref: the oracle's errors of the latest call ([B,Hkv,t_new], NaN where
    no token was written); starts: seq_len of every row before that call.
    band: {(b, h): set of positions} whose routing may differ, carried over
    from earlier calls and extended here.  Returns the updated band.
    rows: optional list of (b, h) to check; all by default.
    abs_k, abs_v: coef_abs_bound of this call's inputs ([B,Hkv,t_new,r]); the
    coefficients this call wrote are checked against 1 ulp + the fp32 bound.
    """
    D = oc.dims
    band = {} if band is None else band
    assert np.array_equal(gc.seq_len, oc.seq_len)
    assert gc.status == oc.status, (gc.status, oc.status)
    rows = rows or [(b, h) for b in range(D.B) for h in range(D.Hkv)]
    for b, h in rows:
        T = int(oc.seq_len[b])
        t0 = int(starts[b])
        # coefficients written by this call: 1 ulp + the fp32 accumulation bound
        for got, want, ab in ((gc.coef_k[b, h, t0:T], oc.coef_k[b, h, t0:T], abs_k),
                              (gc.coef_v[b, h, t0:T], oc.coef_v[b, h, t0:T], abs_v)):
            tol = O.bf16_ulp(np.maximum(np.abs(got), np.abs(want)))
            if ab is not None:
                tol = tol + COEF_ABS_SAFETY * GAMMA_128 * ab[b, h, :T - t0]
            bad = np.abs(got - want) > tol
            assert not bad.any(), f"(b={b},h={h}) {bad.sum()} coefficients off by more than the bound"
        # routed sets: identical outside the band around tau
        eb = e_ref[b, h]
        t_in = np.flatnonzero(~np.isnan(eb) & (np.abs(eb - tau) < BAND))
        bp = band.setdefault((b, h), set())
        bp.update(int(starts[b]) + int(t) for t in t_in)
        rg, ro = set(routed_positions(gc, b, h)), set(routed_positions(oc, b, h))
        assert (rg ^ ro) <= bp, f"(b={b},h={h}) routed sets differ: {sorted(rg ^ ro)[:10]}"
        # the list: ascending positions matching the mask, rows copied bit-exactly
        n = int(gc.full_cnt[b, h])
        idx = gc.full_idx[b, h, :n]
        assert np.all(np.diff(idx) > 0)
        assert set(idx.tolist()) == rg
        o_rows = {int(p): i for i, p in enumerate(oc.full_idx[b, h, :int(oc.full_cnt[b, h])])}
        for i, p in enumerate(idx):
            if int(p) in o_rows:
                j = o_rows[int(p)]
                assert np.array_equal(gc.full_k[b, h, i], oc.full_k[b, h, j])
                assert np.array_equal(gc.full_v[b, h, i], oc.full_v[b, h, j])
        if err_gpu is not None:
            eg = err_gpu[b, h]
            ok = ~np.isnan(e_ref[b, h])
            assert np.array_equal(~np.isnan(eg), ok)
            assert np.abs(eg[ok] - e_ref[b, h][ok]).max(initial=0.0) <= ERR_ATOL
    return band
