"""CUDA library vs the fp64 oracle, element by element, through the C ABI.

Sizes span several projection tiles and decode splits with ragged tails;
the workloads are the tiny GQA-4 case and reduced-size versions of the
Llama-3.1-8B / LLaMA-7B geometries (full sizes are in test_gpu_fullsize.py).
Bars: routed-token sets identical except tokens within 1e-4 of tau,
coefficients within 1 bf16 ulp plus the fp32 dot-product rounding bound,
full-rank rows and list positions exact,
decode output ||o - o_ref||_inf / ||o_ref||_inf <= 2e-3 per call.
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


def _setup(w, seed, T_cap=None, F_cap=None):
    layer = synth.make_layer(w, 0, seed, device=DEV)
    T_cap = T_cap or synth.pad_to(w.T + max(w.t_append, 1), 32)
    D = U.dims_of(w, T_cap, F_cap)
    cache = L.LayerCache(D, layer["U_k"], layer["U_v"], device=DEV)
    oc = O.Cache.empty(U.oracle_dims(D), U.f64(layer["U_k"]), U.f64(layer["U_v"]))
    ws = L.make_workspace(D, DEV)
    return layer, D, cache, oc, ws


def _compress_both(D, cache, oc, K, V, tau, ws, t_new_b=None, band=None):
    starts = oc.seq_len.copy()
    err = U.gpu_compress(D, cache, K, V, tau, ws,
                         t_new_b=None if t_new_b is None else torch.tensor(t_new_b, dtype=torch.int32, device=DEV))
    Kf, Vf = U.f64(K), U.f64(V)
    e_ref, _, _ = O.compress(oc, Kf, Vf, tau, t_new_b=t_new_b)
    torch.cuda.synchronize()
    gc = U.gpu_to_oracle(D, cache)
    band = U.check_compress_parity(gc, oc, e_ref, tau, starts, err_gpu=U.f64(err), band=band,
                                   abs_k=U.coef_abs_bound(oc.U_k, Kf),
                                   abs_v=U.coef_abs_bound(oc.U_v, Vf))
    return gc, band


WORKLOADS = [
    ("tiny", synth.workload(0)),
    ("llama8k_small", synth.workload(1, T=1000, layers=1)),
    ("llama32k_small", synth.workload(2, T=1337, layers=1, t_append=5)),
    ("ragged_small", synth.workload(3, B=4, T=700, ragged_min=300, layers=1)),
    ("mha_small", synth.workload(4, T=600, layers=1)),
]


@pytest.mark.parametrize("name,w", WORKLOADS, ids=[n for n, _ in WORKLOADS])
def test_compress_then_decode(name, w):
    layer, D, cache, oc, ws = _setup(w, seed=11)
    lengths = layer["lengths"].tolist()
    t_new_b = lengths if w.ragged_min else None
    gc, band = _compress_both(D, cache, oc, layer["K"], layer["V"], w.tau, ws, t_new_b=t_new_b)
    routed = int(oc.full_cnt.sum())
    assert routed >= sum(round(w.f_out * n) for n in lengths) * w.Hkv * 0.9
    # decode on the GPU-written cache vs the oracle on the same cache, and vs the oracle's own cache
    out = U.f64(U.gpu_decode(D, cache, layer["q"], ws))
    ref_same = O.decode_attn(gc, U.f64(layer["q"]))
    assert U.out_rel_err(out, ref_same) <= U.OUT_RTOL
    ref_own = O.decode_attn(oc, U.f64(layer["q"]))
    assert U.out_rel_err(out, ref_own) <= U.OUT_RTOL
    # decode-time appends: append one token, then attend (it included), a few times
    if w.t_append:
        for s in range(w.t_append):
            gc, band = _compress_both(D, cache, oc, layer["K_app"][:, s:s + 1],
                                      layer["V_app"][:, s:s + 1], w.tau, ws, band=band)
            out = U.f64(U.gpu_decode(D, cache, layer["q_app"][s], ws))
            assert U.out_rel_err(out, O.decode_attn(gc, U.f64(layer["q_app"][s]))) <= U.OUT_RTOL


@pytest.mark.parametrize("T", [1, 2, 3, 31, 32, 33, 255, 256, 257])
def test_short_and_ragged_lengths(T):
    w = synth.workload(0, T=T)
    layer, D, cache, oc, ws = _setup(w, seed=T, T_cap=synth.pad_to(T + 1, 32))
    gc, _ = _compress_both(D, cache, oc, layer["K"], layer["V"], w.tau, ws)
    out = U.f64(U.gpu_decode(D, cache, layer["q"], ws))
    assert U.out_rel_err(out, O.decode_attn(gc, U.f64(layer["q"]))) <= U.OUT_RTOL


def test_decode_on_oracle_written_cache():
    """Decode alone: the oracle builds the cache, the GPU attends over it."""
    w = synth.workload(1, T=2100, layers=1)
    layer = synth.make_layer(w, 0, 5, device=DEV)
    D = U.dims_of(w, synth.pad_to(w.T, 32))
    oc = O.Cache.empty(U.oracle_dims(D), U.f64(layer["U_k"]), U.f64(layer["U_v"]))
    O.compress(oc, U.f64(layer["K"]), U.f64(layer["V"]), w.tau)
    dims, cache = U.oracle_to_gpu(oc)
    ws = L.make_workspace(dims, DEV)
    out = U.f64(U.gpu_decode(dims, cache, layer["q"], ws))
    assert U.out_rel_err(out, O.decode_attn(oc, U.f64(layer["q"]))) <= U.OUT_RTOL
    # the same workspace serves a second call (tickets were left zeroed)
    out2 = U.f64(U.gpu_decode(dims, cache, layer["q"], ws))
    assert np.array_equal(out, out2)


@pytest.mark.parametrize("tau", [-1.0, 2.0])
def test_all_or_nothing_routed(tau):
    w = synth.workload(1, T=900, layers=1)
    layer, D, cache, oc, ws = _setup(w, seed=3)
    gc, _ = _compress_both(D, cache, oc, layer["K"], layer["V"], tau, ws)
    n = int(gc.full_cnt.sum())
    assert n == (D.B * D.Hkv * w.T if tau < 0 else 0)
    out = U.f64(U.gpu_decode(D, cache, layer["q"], ws))
    assert U.out_rel_err(out, O.decode_attn(gc, U.f64(layer["q"]))) <= U.OUT_RTOL


def test_identity_basis_matches_dense_attention():
    """r = d, U = I: the compressed path must equal dense attention over K, V."""
    B, T, Hkv, Hq, d = 2, 300, 2, 8, 128
    g = torch.Generator(device=DEV).manual_seed(0)
    K = torch.randn(B, T, Hkv, d, generator=g, device=DEV).to(torch.bfloat16)
    V = torch.randn(B, T, Hkv, d, generator=g, device=DEV).to(torch.bfloat16)
    q = torch.randn(B, Hq, d, generator=g, device=DEV).to(torch.bfloat16)
    I = torch.eye(d, device=DEV).expand(Hkv, d, d).to(torch.bfloat16)
    D = L.Dims(B=B, Hq=Hq, Hkv=Hkv, d=d, r_k=d, r_v=d, T_cap=320, F_cap=320)
    cache = L.LayerCache(D, I, I, device=DEV)
    ws = L.make_workspace(D, DEV)
    L.lrkv_compress(D, cache, K, V, 0.3, ws=ws)
    out = U.gpu_decode(D, cache, q, ws)
    ref = torch.nn.functional.scaled_dot_product_attention(
        q.double()[:, :, None], K.double().transpose(1, 2), V.double().transpose(1, 2),
        enable_gqa=True)[:, :, 0]
    assert int(cache.full_cnt.sum()) == 0
    assert U.out_rel_err(U.f64(out), ref.cpu().numpy()) <= 1e-5


def test_empty_and_mixed_batch():
    w = synth.workload(3, B=3, T=200, ragged_min=100, layers=1)
    layer, D, cache, oc, ws = _setup(w, seed=8, T_cap=224)
    t_new_b = [0, 150, 199]
    gc, _ = _compress_both(D, cache, oc, layer["K"], layer["V"], w.tau, ws, t_new_b=t_new_b)
    out = U.f64(U.gpu_decode(D, cache, layer["q"], ws))
    assert not out[0].any()
    assert U.out_rel_err(out, O.decode_attn(gc, U.f64(layer["q"]))) <= U.OUT_RTOL


def test_capacity_overflow_is_reported_and_clamped():
    w = synth.workload(1, T=400, layers=1)
    layer, D, cache, oc, ws = _setup(w, seed=4, T_cap=384, F_cap=5)
    gc, _ = _compress_both(D, cache, oc, layer["K"], layer["V"], w.tau, ws)
    assert gc.status == (L.DEV_FULL_OVERFLOW | L.DEV_SEQ_OVERFLOW)
    assert list(gc.seq_len) == [384] and (gc.full_cnt == 5).all()
    out = U.f64(U.gpu_decode(D, cache, layer["q"], ws))
    assert U.out_rel_err(out, O.decode_attn(gc, U.f64(layer["q"]))) <= U.OUT_RTOL
    # appending to a full sequence drops the token and only raises SEQ_OVERFLOW again
    cache.dev_status.zero_()
    oc.status = 0
    _compress_both(D, cache, oc, layer["K"][:, :1], layer["V"][:, :1], w.tau, ws)


def test_bad_ragged_count_is_clamped():
    w = synth.workload(0, B=2, T=64)
    layer, D, cache, oc, ws = _setup(w, seed=2, T_cap=96)
    L.lrkv_compress(D, cache, layer["K"], layer["V"], w.tau,
                    t_new_b=torch.tensor([70, -3], dtype=torch.int32, device=DEV), ws=ws)
    torch.cuda.synchronize()
    assert int(cache.dev_status[0]) & L.DEV_BAD_COUNT
    assert cache.seq_len.tolist() == [64, 0]


def test_canaries_past_buffers_untouched():
    """Bytes just past every buffer the library writes stay as they were."""
    w = synth.workload(0, T=100)
    layer = synth.make_layer(w, 0, 1, device=DEV)
    D = U.dims_of(w, 128, 16)
    cache = L.LayerCache(D, layer["U_k"], layer["U_v"], device=DEV)
    pad = 4096
    for f in ("coef_k", "coef_v", "route_mask", "full_idx", "full_k", "full_v", "full_cnt", "seq_len"):
        t = getattr(cache, f)
        big = torch.full((t.numel() + pad,), 0x5A5A, dtype=torch.int16 if t.element_size() == 2
                         else torch.int32, device=DEV)
        big[: t.numel()] = 0
        setattr(cache, f, big[: t.numel()].view(t.dtype).view(t.shape))
        setattr(cache, f + "_canary", big)
    ws_n = L.lrkv_workspace_size(D)
    ws_big = torch.full((ws_n + pad,), 0x5A, dtype=torch.uint8, device=DEV)
    ws_big[:ws_n] = 0
    ws = ws_big[:ws_n]
    L.lrkv_compress(D, cache, layer["K"], layer["V"], -1.0, ws=ws)     # everything routed: overflow
    out = torch.empty(w.B, w.Hq, w.d, device=DEV)
    L.lrkv_decode_attn(D, cache, layer["q"], out, ws=ws)
    torch.cuda.synchronize()
    for f in ("coef_k", "coef_v", "route_mask", "full_idx", "full_k", "full_v", "full_cnt", "seq_len"):
        big = getattr(cache, f + "_canary")
        n = getattr(cache, f).numel()
        assert (big[n:] == 0x5A5A).all(), f
    assert (ws_big[ws_n:] == 0x5A).all()
    assert int(cache.dev_status[0]) == L.DEV_FULL_OVERFLOW


def test_small_multi_token_appends_with_ragged_counts():
    """Appends of a few tokens (the fused one-launch path) with ragged counts and a
    nearly full list, interleaved with decode."""
    w = synth.workload(1, B=3, T=300, layers=1)
    layer, D, cache, oc, ws = _setup(w, seed=21, T_cap=352, F_cap=40)
    gc, band = _compress_both(D, cache, oc, layer["K"], layer["V"], w.tau, ws,
                              t_new_b=[300, 150, 290])
    extra = synth.decode_tokens(w, layer["Qk"], layer["Qv"], 7, 21, 0, DEV)
    for counts in ([7, 0, 3], [1, 7, 7], [7, 7, 7]):
        gc, band = _compress_both(D, cache, oc, extra[0], extra[1], w.tau, ws, t_new_b=counts,
                                  band=band)
        out = U.f64(U.gpu_decode(D, cache, layer["q"], ws))
        assert U.out_rel_err(out, O.decode_attn(gc, U.f64(layer["q"]))) <= U.OUT_RTOL


def test_prefill_in_two_parts_unaligned_start():
    """Two prefill calls, the second starting mid mask word, with several
    128-token tiles per projection CTA (stage and accumulator buffers reused)."""
    w = synth.workload(1, B=2, T=3000, layers=1)
    layer, D, cache, oc, ws = _setup(w, seed=9, T_cap=3008)
    K, V = layer["K"], layer["V"]
    cut = 1237
    gc, band = _compress_both(D, cache, oc, K[:, :cut].contiguous(), V[:, :cut].contiguous(),
                              w.tau, ws, t_new_b=[cut, 1000])
    gc, band = _compress_both(D, cache, oc, K[:, cut:].contiguous(), V[:, cut:].contiguous(),
                              w.tau, ws, t_new_b=[3000 - cut, 1500], band=band)
    assert list(gc.seq_len) == [3000, 2500]
    out = U.f64(U.gpu_decode(D, cache, layer["q"], ws))
    assert U.out_rel_err(out, O.decode_attn(gc, U.f64(layer["q"]))) <= U.OUT_RTOL


def test_scatter_with_runs_of_tiles_per_cta():
    """A prefill of 4 x 8 (b, kv head) pairs x 150 tiles of 128 tokens: more
    than twice a wave of 128-thread CTAs on a 148-SM part, so the scatter pass
    gives each CTA a run of tiles.  Ragged rows, a start mid mask word, and a
    list that fills up partway through the runs (FULL_OVERFLOW)."""
    w = synth.workload(1, B=4, T=19237, layers=1)
    layer, D, cache, oc, ws = _setup(w, seed=53, T_cap=19264, F_cap=1200)
    K, V = layer["K"], layer["V"]
    cut = 37
    gc, band = _compress_both(D, cache, oc, K[:, :cut].contiguous(), V[:, :cut].contiguous(),
                              w.tau, ws)
    gc, band = _compress_both(D, cache, oc, K[:, cut:].contiguous(), V[:, cut:].contiguous(),
                              w.tau, ws, t_new_b=[19200, 18000, 19100, 17500], band=band)
    assert gc.status & L.DEV_FULL_OVERFLOW
    assert list(gc.seq_len) == [19237, 18037, 19137, 17537]
    out = U.f64(U.gpu_decode(D, cache, layer["q"], ws))
    assert U.out_rel_err(out, O.decode_attn(gc, U.f64(layer["q"]))) <= U.OUT_RTOL


@pytest.mark.parametrize("Hq,Hkv,r_k,r_v", [(16, 8, 48, 80), (4, 2, 64, 64), (6, 2, 48, 64),
                                            (16, 2, 32, 32), (20, 4, 64, 96), (8, 8, 32, 48),
                                            (6, 2, 32, 48), (16, 2, 32, 48)],
                         ids=["g2_48_80", "g2_64_64", "g3_stream", "g8_stream_two_passes",
                              "g5_stream_two_passes", "g1_rank_pair_simple", "g3_simple", "g8_simple"])
def test_group_sizes_and_rank_pairs(Hq, Hkv, r_k, r_v):
    """GQA groups of 1, 2, 3, 5 and 8 query heads: the streaming kernel takes
    any group in launches of up to 4 heads (3: one launch with an idle head;
    5, 8: two launches); a rank pair outside its instantiations (32/48) goes to
    the CUDA-core kernel, at groups of 1, 3 and 8."""
    w = synth.workload(1, Hq=Hq, Hkv=Hkv, r_k=r_k, r_v=r_v, T=900, layers=1)
    layer, D, cache, oc, ws = _setup(w, seed=13)
    gc, band = _compress_both(D, cache, oc, layer["K"], layer["V"], w.tau, ws)
    extra = synth.decode_tokens(w, layer["Qk"], layer["Qv"], 2, 13, 0, DEV)
    gc, band = _compress_both(D, cache, oc, extra[0][:, :1].contiguous(), extra[1][:, :1].contiguous(),
                              w.tau, ws, band=band)
    out = U.f64(U.gpu_decode(D, cache, layer["q"], ws))
    assert U.out_rel_err(out, O.decode_attn(gc, U.f64(layer["q"]))) <= U.OUT_RTOL


@pytest.mark.parametrize("Hq,Hkv,r_k,r_v", [(32, 8, 64, 96), (24, 8, 64, 96), (4, 4, 48, 64)])
def test_capacity_far_above_the_live_length(Hq, Hkv, r_k, r_v):
    """A cache allocated for 16384 positions that holds 600: the decode splits
    follow the live length (the grid is sized for the capacity), with the
    streaming kernel at GQA 4, MHA and GQA 3 (a launch of 4 heads, one idle);
    then a fused append + decode step on the same cache."""
    w = synth.workload(1, Hq=Hq, Hkv=Hkv, r_k=r_k, r_v=r_v, T=600, layers=1)
    layer, D, cache, oc, ws = _setup(w, seed=19, T_cap=16384, F_cap=4096)
    gc, band = _compress_both(D, cache, oc, layer["K"], layer["V"], w.tau, ws)
    out = U.f64(U.gpu_decode(D, cache, layer["q"], ws))
    assert U.out_rel_err(out, O.decode_attn(gc, U.f64(layer["q"]))) <= U.OUT_RTOL
    Ka, Va = synth.decode_tokens(w, layer["Qk"], layer["Qv"], 1, 19, 0, DEV)
    o2 = torch.empty(D.B, D.Hq, D.d, dtype=torch.float32, device=DEV)
    L.lrkv_append_decode_attn(D, cache, Ka.contiguous(), Va.contiguous(), w.tau, layer["q"], o2, ws=ws)
    O.compress(oc, U.f64(Ka), U.f64(Va), w.tau)
    torch.cuda.synchronize()
    gc = U.gpu_to_oracle(D, cache)
    assert list(gc.seq_len) == [601] and gc.status == 0
    assert U.out_rel_err(U.f64(o2), O.decode_attn(gc, U.f64(layer["q"]))) <= U.OUT_RTOL


def test_degenerate_zero_rows_no_list_exact_fill():
    """All-zero key/value rows (e := 0, never routed), a key-only zero row, a
    cache with no full-rank list (F_cap = 0: every routed token overflows and
    stays compressed), and a prefill that fills T_cap exactly."""
    w = synth.workload(0, T=512)
    layer, D, cache, oc, ws = _setup(w, seed=17, T_cap=512, F_cap=0)
    K, V = layer["K"].clone(), layer["V"].clone()
    K[:, 100:140] = 0
    V[:, 100:140] = 0
    K[:, 300] = 0
    for f in ("full_idx", "full_k", "full_v"):
        getattr(cache, f).fill_(0x3C3C)
    gc, _ = _compress_both(D, cache, oc, K, V, w.tau, ws)
    assert list(gc.seq_len) == [512]
    assert gc.status == L.DEV_FULL_OVERFLOW and int(gc.full_cnt.sum()) == 0
    assert not gc.route_mask.any()
    for f in ("full_idx", "full_k", "full_v"):
        assert (getattr(cache, f) == 0x3C3C).all(), f
    assert not gc.coef_k[0, 0, 100:140].any() and not gc.coef_v[0, 0, 100:140].any()
    out = U.f64(U.gpu_decode(D, cache, layer["q"], ws))
    assert U.out_rel_err(out, O.decode_attn(gc, U.f64(layer["q"]))) <= U.OUT_RTOL
    # one more token: the sequence is full, the token is dropped
    cache.dev_status.zero_()
    oc.status = 0
    gc, _ = _compress_both(D, cache, oc, K[:, :1].contiguous(), V[:, :1].contiguous(), w.tau, ws)
    assert gc.status == L.DEV_SEQ_OVERFLOW and list(gc.seq_len) == [512]
