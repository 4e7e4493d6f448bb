"""lrkv_append_decode_attn (append one token per row, then attend, in one
launch) vs the fp64 oracle running compress then decode, through the C ABI.

The same bars as the separate calls: coefficients within 1 bf16 ulp plus the
fp32 dot-product bound, routed sets identical except tokens within 1e-4 of
tau, list rows exact and in position order, the error output within 5e-5,
seq_len and status words equal, and each step's output within
||o - o_ref||_inf / ||o_ref||_inf <= 2e-3 of the oracle attending over the
cache after the append.  Also: the fused call and the two separate calls
leave the same cache, rows with no token, full sequences, a full list, a
split grid with no CTA to spare for the append, and a shape the streaming
kernel does not cover (two launches).
"""
import numpy as np
import pytest
import torch

import oracle as O
import synth
import decode_attention_lrkv_b200 as L
from tests import lrkv_testutil as U
from tests.test_gpu_parity import WORKLOADS, _compress_both, _setup

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _fused_both(D, cache, oc, k, v, q, tau, ws, t_new_b=None, band=None):
    """One fused step on the GPU, compress + decode in the oracle; checks both."""
    starts = oc.seq_len.copy()
    err = torch.full((D.B, D.Hkv, 1), float("nan"), device=DEV)
    out = torch.empty(D.B, D.Hq, D.d, dtype=torch.float32, device=DEV)
    tb = None if t_new_b is None else torch.tensor(t_new_b, dtype=torch.int32, device=DEV)
    L.lrkv_append_decode_attn(D, cache, k, v, tau, q, out, t_new_b=tb, err_out=err, ws=ws)
    kf, vf = U.f64(k), U.f64(v)
    e_ref, _, _ = O.compress(oc, kf, vf, tau, t_new_b=t_new_b)
    torch.cuda.synchronize()
    gc = U.gpu_to_oracle(D, cache)
    band = U.check_compress_parity(gc, oc, e_ref, tau, starts, err_gpu=U.f64(err), band=band,
                                   abs_k=U.coef_abs_bound(oc.U_k, kf),
                                   abs_v=U.coef_abs_bound(oc.U_v, vf))
    o = U.f64(out)
    qf = U.f64(q)
    assert U.out_rel_err(o, O.decode_attn(gc, qf)) <= U.OUT_RTOL
    assert U.out_rel_err(o, O.decode_attn(oc, qf)) <= U.OUT_RTOL
    return gc, band, o


@pytest.mark.parametrize("name,w", WORKLOADS, ids=[n for n, _ in WORKLOADS])
def test_fused_steps_match_oracle(name, w):
    layer, D, cache, oc, ws = _setup(w, seed=23, T_cap=synth.pad_to(w.T + 8, 32))
    lengths = layer["lengths"].tolist()
    t_new_b = lengths if w.ragged_min else None
    _, band = _compress_both(D, cache, oc, layer["K"], layer["V"], w.tau, ws, t_new_b=t_new_b)
    Ka, Va = synth.decode_tokens(w, layer["Qk"], layer["Qv"], 6, 23, 0, DEV)
    qs = synth.decode_queries(w, 6, 23, 0, DEV)
    for s in range(6):
        _, band, _ = _fused_both(D, cache, oc, Ka[:, s:s + 1].contiguous(),
                                 Va[:, s:s + 1].contiguous(), qs[s], w.tau, ws, band=band)


def test_fused_equals_two_calls():
    """Same cache after the fused call as after lrkv_compress + lrkv_decode_attn."""
    w = synth.workload(2, T=1337, layers=1)
    layer = synth.make_layer(w, 0, 29, device=DEV)
    D = U.dims_of(w, synth.pad_to(w.T + 8, 32))
    caches = [L.LayerCache(D, layer["U_k"], layer["U_v"], device=DEV) for _ in range(2)]
    wss = [L.make_workspace(D, DEV) for _ in range(2)]
    for c, ws in zip(caches, wss):
        L.lrkv_compress(D, c, layer["K"], layer["V"], w.tau, ws=ws)
    Ka, Va = synth.decode_tokens(w, layer["Qk"], layer["Qv"], 4, 29, 0, DEV)
    qs = synth.decode_queries(w, 4, 29, 0, DEV)
    for s in range(4):
        k, v = Ka[:, s:s + 1].contiguous(), Va[:, s:s + 1].contiguous()
        o1 = torch.empty(D.B, D.Hq, D.d, device=DEV)
        L.lrkv_append_decode_attn(D, caches[0], k, v, w.tau, qs[s], o1, ws=wss[0])
        L.lrkv_compress(D, caches[1], k, v, w.tau, ws=wss[1])
        o2 = U.gpu_decode(D, caches[1], qs[s], wss[1])
        torch.cuda.synchronize()
        for f in ("seq_len", "full_cnt", "route_mask", "full_idx", "full_k", "full_v", "dev_status"):
            assert torch.equal(getattr(caches[0], f), getattr(caches[1], f)), f
        # coefficients: both fp32-accurate, rounded to bf16: within one ulp of each other
        for f in ("coef_k", "coef_v"):
            a, b = U.f64(getattr(caches[0], f)), U.f64(getattr(caches[1], f))
            assert (np.abs(a - b) <= O.bf16_ulp(np.maximum(np.abs(a), np.abs(b)))).all(), f
        assert U.out_rel_err(U.f64(o1), U.f64(o2)) <= U.OUT_RTOL


def test_fused_rows_without_token_and_full_sequences():
    """t_new_b of 0 attends only; a row at T_cap drops its token (SEQ_OVERFLOW)."""
    w = synth.workload(3, B=4, T=300, ragged_min=200, layers=1)
    layer, D, cache, oc, ws = _setup(w, seed=31, T_cap=320)
    lengths = layer["lengths"].tolist()
    lengths[2] = 320                       # row 2 fills the cache
    K = torch.cat([layer["K"], layer["K"][:, :20]], dim=1).contiguous()
    V = torch.cat([layer["V"], layer["V"][:, :20]], dim=1).contiguous()
    _, band = _compress_both(D, cache, oc, K, V, w.tau, ws, t_new_b=lengths)
    Ka, Va = synth.decode_tokens(w, layer["Qk"], layer["Qv"], 3, 31, 0, DEV)
    qs = synth.decode_queries(w, 3, 31, 0, DEV)
    for s, tb in enumerate(([1, 0, 1, 1], [0, 1, 1, 0], [1, 1, 0, 1])):
        cache.dev_status.zero_()
        oc.status = 0
        gc, band, _ = _fused_both(D, cache, oc, Ka[:, s:s + 1].contiguous(),
                                  Va[:, s:s + 1].contiguous(), qs[s], w.tau, ws, t_new_b=tb,
                                  band=band)
        assert (gc.status & L.DEV_SEQ_OVERFLOW) == (L.DEV_SEQ_OVERFLOW if tb[2] else 0)
    assert int(gc.seq_len[2]) == 320


@pytest.mark.parametrize("tau", [-1.0, 2.0])
def test_fused_all_or_nothing_routed_and_full_list(tau):
    """Every new token routed (tau < 0) until the list is full, or none routed."""
    w = synth.workload(1, T=500, layers=1)
    layer, D, cache, oc, ws = _setup(w, seed=37, T_cap=544, F_cap=502)
    _, band = _compress_both(D, cache, oc, layer["K"], layer["V"], tau, ws)
    Ka, Va = synth.decode_tokens(w, layer["Qk"], layer["Qv"], 4, 37, 0, DEV)
    qs = synth.decode_queries(w, 4, 37, 0, DEV)
    for s in range(4):
        cache.dev_status.zero_()
        oc.status = 0
        gc, band, _ = _fused_both(D, cache, oc, Ka[:, s:s + 1].contiguous(),
                                  Va[:, s:s + 1].contiguous(), qs[s], tau, ws, band=band)
        if tau < 0:
            assert (gc.full_cnt == min(500 + s + 1, 502)).all()
            assert (gc.status & L.DEV_FULL_OVERFLOW) == (L.DEV_FULL_OVERFLOW if s >= 2 else 0)
        else:
            assert (gc.full_cnt == 0).all()


@pytest.mark.parametrize("T", [1, 31, 32, 33, 127, 128, 129, 383, 384, 385])
def test_fused_at_split_boundaries(T):
    """The new position opens a new split exactly when T is a multiple of the split length."""
    w = synth.workload(1, T=T, layers=1)
    layer, D, cache, oc, ws = _setup(w, seed=41 + T, T_cap=synth.pad_to(T + 3, 32))
    _, band = _compress_both(D, cache, oc, layer["K"], layer["V"], w.tau, ws)
    Ka, Va = synth.decode_tokens(w, layer["Qk"], layer["Qv"], 2, 41, 0, DEV)
    qs = synth.decode_queries(w, 2, 41, 0, DEV)
    for s in range(2):
        _, band, _ = _fused_both(D, cache, oc, Ka[:, s:s + 1].contiguous(),
                                 Va[:, s:s + 1].contiguous(), qs[s], w.tau, ws, band=band)


def test_fused_when_the_split_grid_has_no_spare_cta():
    """B * Hkv = 64 sequences-heads with T_cap = 8224: the split model gives a
    full cache two splits of at most 8192 positions, and a cached length past
    8192 needs both of them as well, so the fused call's grid holds a third CTA
    for the append.  Two steps at cached lengths 8222 and 8223 attend to every
    position and keep each (b, kv head)'s records apart."""
    w = synth.workload(1, B=8, T=8222, layers=1)
    layer, D, cache, oc, ws = _setup(w, seed=47, T_cap=8224, F_cap=2048)
    _, band = _compress_both(D, cache, oc, layer["K"], layer["V"], w.tau, ws)
    Ka, Va = synth.decode_tokens(w, layer["Qk"], layer["Qv"], 2, 47, 0, DEV)
    qs = synth.decode_queries(w, 2, 47, 0, DEV)
    for s in range(2):
        gc, band, _ = _fused_both(D, cache, oc, Ka[:, s:s + 1].contiguous(),
                                  Va[:, s:s + 1].contiguous(), qs[s], w.tau, ws, band=band)
    assert (gc.seq_len == 8224).all()
    out = torch.empty(D.B, D.Hq, D.d, dtype=torch.float32, device=DEV)   # and a plain decode of the full cache
    L.lrkv_decode_attn(D, cache, qs[0], out, ws=ws)
    torch.cuda.synchronize()
    assert U.out_rel_err(U.f64(out), O.decode_attn(oc, U.f64(qs[0]))) <= U.OUT_RTOL


def test_fused_on_an_empty_cache():
    w = synth.workload(0, T=4)
    layer, D, cache, oc, ws = _setup(w, seed=43, T_cap=32)
    band = None
    for s in range(3):
        _, band, _ = _fused_both(D, cache, oc, layer["K"][:, s:s + 1].contiguous(),
                                 layer["V"][:, s:s + 1].contiguous(), layer["q"], w.tau, ws,
                                 band=band)


@pytest.mark.parametrize("Hq,r_k,r_v", [(6, 32, 48), (6, 64, 96), (16, 64, 96), (10, 48, 64)],
                         ids=["g3_no_streaming_kernel", "g3_one_launch", "g8_two_launches", "g5_two_launches"])
def test_fused_other_group_sizes(Hq, r_k, r_v):
    """Groups of 3, 5 and 8 query heads per kv head: the streaming kernel runs
    the fused step in launches of 4 heads, the first of which appends (later
    launches read the appended token); a rank pair it has no instantiation for
    (32/48) runs the two launches the call fuses."""
    w = synth.workload(1, T=300, layers=1, r_k=r_k, r_v=r_v)
    layer = synth.make_layer(w, 0, 47, device=DEV)
    Hkv = 2
    D = L.Dims(B=1, Hq=Hq, Hkv=Hkv, d=128, r_k=r_k, r_v=r_v, T_cap=320, F_cap=320)
    U_k, U_v = layer["U_k"][:Hkv].contiguous(), layer["U_v"][:Hkv].contiguous()
    cache = L.LayerCache(D, U_k, U_v, device=DEV)
    oc = O.Cache.empty(U.oracle_dims(D), U.f64(U_k), U.f64(U_v))
    ws = L.make_workspace(D, DEV)
    K, V = layer["K"][:, :, :Hkv].contiguous(), layer["V"][:, :, :Hkv].contiguous()
    _, band = _compress_both(D, cache, oc, K, V, w.tau, ws)
    g = torch.Generator(device=DEV).manual_seed(47)
    for s in range(2):
        k = torch.randn(1, 1, Hkv, 128, generator=g, device=DEV).to(torch.bfloat16)
        v = torch.randn(1, 1, Hkv, 128, generator=g, device=DEV).to(torch.bfloat16)
        q = torch.randn(1, Hq, 128, generator=g, device=DEV).to(torch.bfloat16)
        _, band, _ = _fused_both(D, cache, oc, k, v, q, w.tau, ws, band=band)
