"""Quantised coefficient caches (int8 and int4 codes with per-row scales)
through the CUDA library vs the fp64 oracle (oracle/coef_quant.py).

KVQuant record (sub-8-bit codes with per-vector scales) and NOVA-KV summary
(fixed-width codes read inside attention), applied to this cache's stored
rows by reading R21: s = amax|bf16(c)| / Q, q = round_half_even(bf16(c) / s),
IEEE fp32 steps.  The write path (prefill projection, small appends, fused
append) quantises as it stores; the decode reads codes times scales.

Bars:
  - codes and scales bit-exact against quantize_coef of the bf16 rows that the
    same write calls store in a bf16 cache (the GPU's own fp32 projections: the
    quantiser takes its integer decisions on exactly the values it quantises);
    that bf16 cache is itself checked against the oracle as in the plain tests
    (1 bf16 ulp plus the fp32 accumulation bound, reading R14);
  - routed sets, list rows, lengths and status identical to the bf16 cache's
    (and to the oracle's outside 1e-4 of tau);
  - decode ||o - o_ref||_inf / ||o_ref||_inf <= 2e-3 against the oracle's plain
    decode over the dequantised rows (decode_attn_quant), on the GPU-written
    cache and on an oracle-written one.
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


def gpu_codes(D, cache):
    """The GPU cache's codes (int8 values [B,Hkv,T_cap,r]) and scales."""
    def codes(t):
        a = t.cpu().numpy()
        return a.view(np.int8) if D.bits == 8 else O.unpack_int4(a)
    return dict(qk=codes(cache.coef_k), sk=cache.scale_k.cpu().numpy(),
                qv=codes(cache.coef_v), sv=cache.scale_v.cpu().numpy())


def gpu_quant_to_oracle(D, cache):
    """An oracle cache holding the GPU's state, coefficients dequantised from its
    codes (what the decode reads), and the codes themselves."""
    c = O.Cache.empty(U.oracle_dims(D), U.f64(cache.U_k), U.f64(cache.U_v))
    cd = gpu_codes(D, cache)
    c.coef_k[:] = O.dequantize_coef(cd["qk"], cd["sk"])
    c.coef_v[:] = O.dequantize_coef(cd["qv"], cd["sv"])
    c.route_mask[:] = cache.route_mask.cpu().numpy().view(np.uint32)
    if D.F_cap:
        c.full_idx[:] = cache.full_idx.cpu().numpy()[:, :, :D.F_cap]
        c.full_k[:] = U.f64(cache.full_k)[:, :, :D.F_cap]
        c.full_v[:] = U.f64(cache.full_v)[:, :, :D.F_cap]
    c.full_cnt[:] = cache.full_cnt.cpu().numpy()
    c.seq_len[:] = cache.seq_len.cpu().numpy()
    c.status = int(cache.dev_status[0].item()) & 0xFFFFFFFF
    return c, cd


def _step(Db, Dq, cb, cq, oc, K, V, tau, wsb, wsq, bits, band, fused_q=None, t_new_b=None):
    """One write call on the bf16 cache cb, the quantised cache cq and the oracle
    (lrkv_compress, or the fused append + decode when fused_q is given), checked;
    returns (cq's state as an oracle cache, band, fused output or None)."""
    starts = oc.seq_len.copy()
    outs = []
    for D, c, ws in ((Db, cb, wsb), (Dq, cq, wsq)):
        if fused_q is None:
            tb = None if t_new_b is None else torch.tensor(t_new_b, dtype=torch.int32, device=DEV)
            L.lrkv_compress(D, c, K, V, tau, t_new_b=tb, ws=ws)
        else:
            o = torch.empty(D.B, D.Hq, D.d, dtype=torch.float32, device=DEV)
            L.lrkv_append_decode_attn(D, c, K, V, tau, fused_q, o, ws=ws)
            outs.append(o)
    Kf, Vf = U.f64(K), U.f64(V)
    e_ref, _, _ = O.compress(oc, Kf, Vf, tau, t_new_b=t_new_b)
    torch.cuda.synchronize()
    gb = U.gpu_to_oracle(Db, cb)
    band = U.check_compress_parity(gb, oc, e_ref, tau, starts, band=band,
                                   abs_k=U.coef_abs_bound(oc.U_k, Kf), abs_v=U.coef_abs_bound(oc.U_v, Vf))
    gq, gcd = gpu_quant_to_oracle(Dq, cq)
    for f in ("route_mask", "full_idx", "full_k", "full_v", "full_cnt", "seq_len"):
        assert np.array_equal(getattr(gq, f), getattr(gb, f)), f
    assert gq.status == gb.status
    want = O.quantize_cache(gb, bits)   # the quantiser on the bf16 rows the GPU computed
    for b in range(Dq.B):
        p0, p1 = int(starts[b]), int(oc.seq_len[b])
        for key in ("qk", "sk", "qv", "sv"):
            assert np.array_equal(gcd[key][b, :, p0:p1], want[key][b, :, p0:p1]), (key, b)
    return gq, band, (outs[1] if outs else None)


WORKLOADS = [
    ("llama8k_small", synth.workload(1, T=1000, layers=1)),
    ("mha_small", synth.workload(4, T=700, layers=1)),
    ("llama32k_small", synth.workload(2, T=900, layers=1)),
    ("ragged_small", synth.workload(3, B=3, T=600, ragged_min=250, layers=1)),
    ("tiny", synth.workload(0)),
    ("gqa3", synth.workload(1, Hq=24, T=500, layers=1)),
    ("cuda_cores_32_48", synth.workload(1, r_k=32, r_v=48, T=500, layers=1)),
]


@pytest.mark.parametrize("bits", [8, 4])
@pytest.mark.parametrize("name,w", WORKLOADS, ids=[n for n, _ in WORKLOADS])
def test_quantised_cache_write_and_decode(name, w, bits):
    layer = synth.make_layer(w, 0, 71, device=DEV)
    T_cap = synth.pad_to(w.T + 16, 32)
    Db, Dq = U.dims_of(w, T_cap), U.dims_of(w, T_cap, coef_bits=bits)
    cb = L.LayerCache(Db, layer["U_k"], layer["U_v"], device=DEV)
    cq = L.LayerCache(Dq, layer["U_k"], layer["U_v"], device=DEV)
    oc = O.Cache.empty(U.oracle_dims(Db), U.f64(layer["U_k"]), U.f64(layer["U_v"]))
    wsb, wsq = L.make_workspace(Db, DEV), L.make_workspace(Dq, DEV)
    lengths = layer["lengths"].tolist()
    band = {}
    step = lambda K, V, **kw: _step(Db, Dq, cb, cq, oc, K, V, w.tau, wsb, wsq, bits, band, **kw)
    gq, band, _ = step(layer["K"], layer["V"], t_new_b=lengths if w.ragged_min else None)
    q = layer["q"]
    out = U.f64(U.gpu_decode(Dq, cq, q, wsq))
    assert U.out_rel_err(out, O.decode_attn(gq, U.f64(q))) <= U.OUT_RTOL
    assert U.out_rel_err(out, O.decode_attn_quant(oc, O.quantize_cache(oc, bits), U.f64(q))) <= U.OUT_RTOL
    # small appends (3 tokens, then 1), then two fused append + decode steps
    Ka, Va = synth.decode_tokens(w, layer["Qk"], layer["Qv"], 6, 71, 0, DEV)
    gq, band, _ = step(Ka[:, :3].contiguous(), Va[:, :3].contiguous())
    gq, band, _ = step(Ka[:, 3:4].contiguous(), Va[:, 3:4].contiguous())
    qs = synth.decode_queries(w, 2, 71, 0, DEV)
    for s in range(2):
        gq, band, o = step(Ka[:, 4 + s:5 + s].contiguous(), Va[:, 4 + s:5 + s].contiguous(), fused_q=qs[s])
        assert U.out_rel_err(U.f64(o), O.decode_attn(gq, U.f64(qs[s]))) <= U.OUT_RTOL
        assert U.out_rel_err(U.f64(o), O.decode_attn_quant(oc, O.quantize_cache(oc, bits),
                                                           U.f64(qs[s]))) <= U.OUT_RTOL


@pytest.mark.parametrize("bits", [8, 4])
def test_decode_on_oracle_quantised_cache(bits):
    """Decode alone: the oracle writes and quantises the cache, the GPU reads its codes."""
    w = synth.workload(1, T=2100, layers=1)
    layer = synth.make_layer(w, 0, 73, device=DEV)
    D = U.dims_of(w, synth.pad_to(w.T, 32), coef_bits=bits)
    oc = O.Cache.empty(U.oracle_dims(D), U.f64(layer["U_k"]), U.f64(layer["U_v"]))
    O.compress(oc, U.f64(layer["K"]), U.f64(layer["V"]), w.tau)
    ocd = O.quantize_cache(oc, bits)
    _, bf = U.oracle_to_gpu(oc)                     # the list, mask and lengths
    cache = L.LayerCache(D, layer["U_k"], layer["U_v"], device=DEV)
    for f in ("route_mask", "full_idx", "full_k", "full_v", "full_cnt", "seq_len"):
        getattr(cache, f).copy_(getattr(bf, f))
    pack = (lambda a: a.view(np.uint8)) if bits == 8 else O.pack_int4
    cache.coef_k.copy_(torch.from_numpy(np.ascontiguousarray(pack(ocd["qk"]))))
    cache.coef_v.copy_(torch.from_numpy(np.ascontiguousarray(pack(ocd["qv"]))))
    cache.scale_k.copy_(torch.from_numpy(ocd["sk"]))
    cache.scale_v.copy_(torch.from_numpy(ocd["sv"]))
    ws = L.make_workspace(D, DEV)
    out = U.f64(U.gpu_decode(D, cache, layer["q"], ws))
    ref = O.decode_attn_quant(oc, ocd, U.f64(layer["q"]))
    assert U.out_rel_err(out, ref) <= U.OUT_RTOL
    # the code-space form of the oracle agrees with its plain form
    assert U.out_rel_err(O.decode_attn_quant_coef(oc, ocd, U.f64(layer["q"])), ref) <= 1e-12


@pytest.mark.parametrize("bits", [8, 4])
def test_value_scales_spanning_many_octaves(bits):
    """Row value scales that jump by tens of octaves along the sequence (2^-40,
    then 1, then 2^20 times the quantiser's): the int8 value sums run on f16
    operands under a per-warp power-of-two scale that later tiles must lower.
    The decode still matches the oracle's over the same codes and scales."""
    w = synth.workload(1, T=2100, layers=1)
    layer = synth.make_layer(w, 0, 75, device=DEV)
    D = U.dims_of(w, synth.pad_to(w.T, 32), coef_bits=bits)
    oc = O.Cache.empty(U.oracle_dims(D), U.f64(layer["U_k"]), U.f64(layer["U_v"]))
    O.compress(oc, U.f64(layer["K"]), U.f64(layer["V"]), w.tau)
    ocd = O.quantize_cache(oc, bits)
    sv = ocd["sv"].astype(np.float64)
    sv[:, :, :700] *= 2.0 ** -40
    sv[:, :, 1400:] *= 2.0 ** 20
    ocd["sv"] = sv.astype(np.float32)
    _, bf = U.oracle_to_gpu(oc)
    cache = L.LayerCache(D, layer["U_k"], layer["U_v"], device=DEV)
    for f in ("route_mask", "full_idx", "full_k", "full_v", "full_cnt", "seq_len"):
        getattr(cache, f).copy_(getattr(bf, f))
    pack = (lambda a: a.view(np.uint8)) if bits == 8 else O.pack_int4
    cache.coef_k.copy_(torch.from_numpy(np.ascontiguousarray(pack(ocd["qk"]))))
    cache.coef_v.copy_(torch.from_numpy(np.ascontiguousarray(pack(ocd["qv"]))))
    cache.scale_k.copy_(torch.from_numpy(ocd["sk"]))
    cache.scale_v.copy_(torch.from_numpy(ocd["sv"]))
    ws = L.make_workspace(D, DEV)
    # queries that weight the sequence's three parts alike: mostly the
    # full-rank rows and the 2^20-scaled part matter, yet the first part's
    # tiles (scale 2^-40) come first for most warps
    out = U.f64(U.gpu_decode(D, cache, layer["q"], ws))
    ref = O.decode_attn_quant(oc, ocd, U.f64(layer["q"]))
    assert np.isfinite(out).all()
    assert U.out_rel_err(out, ref) <= U.OUT_RTOL
