"""CUDA library vs the fp64 oracle at the benchmark's full sizes.

One layer of each benchmark workload at its full context (Llama-3.1-8B
geometry at 8K and 32K, the batch-16 ragged 8K-16K case and the LLaMA-7B MHA
case at 131072), with the cache capacity bench.py uses, so the kernels run in
the launch configuration bench.py times: a prefill through lrkv_compress,
three one-token appends, then one decode.  The oracle cannot redo whole
layers in seconds, so sampled (batch row, kv head) pairs are recomputed one
by one and compared element by element (then two more steps through the fused
append + decode call, the launch bench.py times, are checked the same way):
  - every coefficient of the head: 1 bf16 ulp + the fp32 accumulation bound;
  - the routed set: identical except tokens within 1e-4 of tau;
  - the full-rank list: ascending positions, rows bit-exact, length;
  - decode output of the head's query heads: ||o - o_ref||_inf / ||o_ref||_inf
    <= 2e-3, the oracle attending over the GPU-written cache.
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
# bench.py's cache capacity: the context plus four passes of its default
# 100 timed + 5 warm-up decode steps, plus one
BENCH_EXTRA = 4 * (100 + 5) + 1
N_APPEND = 3


def _oracle_head(D, U_k1, U_v1, K, V, tau, n_b, appends):
    """The oracle's cache for one (batch row, kv head), built call by call.

    U_k1, U_v1: [1, d, r]; K, V and the appended rows: [1, t, 1, d]."""
    od = O.Dims(B=1, Hq=D.Hq // D.Hkv, Hkv=1, d=D.d, r_k=D.r_k, r_v=D.r_v, T_cap=D.T_cap,
                F_cap=D.F_cap)
    oc = O.Cache.empty(od, U_k1, U_v1)
    e_all = []
    e, _, _ = O.compress(oc, K, V, tau, t_new_b=[n_b])
    e_all.append(e[0, 0, :n_b])
    for Ka, Va in appends:
        e, _, _ = O.compress(oc, Ka, Va, tau)
        e_all.append(e[0, 0])
    return oc, np.concatenate(e_all)


def _gpu_head(D, cache, b, h):
    """The GPU cache's (b, h) slice as a one-head oracle cache."""
    od = O.Dims(B=1, Hq=D.Hq // D.Hkv, Hkv=1, d=D.d, r_k=D.r_k, r_v=D.r_v, T_cap=D.T_cap,
                F_cap=D.F_cap)
    c = O.Cache.empty(od, U.f64(cache.U_k[h:h + 1]), U.f64(cache.U_v[h:h + 1]))
    c.coef_k[0, 0] = U.f64(cache.coef_k[b, h])
    c.coef_v[0, 0] = U.f64(cache.coef_v[b, h])
    c.route_mask[0, 0] = cache.route_mask[b, h].cpu().numpy().view(np.uint32)
    c.full_idx[0, 0] = cache.full_idx[b, h].cpu().numpy()
    c.full_k[0, 0] = U.f64(cache.full_k[b, h])
    c.full_v[0, 0] = U.f64(cache.full_v[b, h])
    c.full_cnt[0, 0] = int(cache.full_cnt[b, h])
    c.seq_len[0] = int(cache.seq_len[b])
    return c


WORKLOADS = [(i, synth.workload(i, layers=1)) for i in (1, 2, 3, 4)]


def bench_f_cap(wi, T_cap):
    """bench.py's full-rank list capacity: all positions on the 32K workload (81%
    routed), a quarter of them elsewhere (7-11% routed)."""
    return T_cap if wi == 2 else synth.pad_to(T_cap // 4, 32)


@pytest.mark.parametrize("wi,w", WORKLOADS, ids=[w.name for _, w in WORKLOADS])
def test_full_size_sampled_heads(wi, w):
    seed = 31 + wi
    layer = synth.make_layer(w, 0, seed, device=DEV)
    T_cap = synth.pad_to(w.T + BENCH_EXTRA, 32)
    D = U.dims_of(w, T_cap, bench_f_cap(wi, T_cap))
    cache = L.LayerCache(D, layer["U_k"], layer["U_v"], device=DEV)
    ws = L.make_workspace(D, DEV)
    lengths = layer["lengths"].tolist()
    t_new_b = torch.tensor(lengths, dtype=torch.int32, device=DEV) if w.ragged_min else None
    L.lrkv_compress(D, cache, layer["K"], layer["V"], w.tau, t_new_b=t_new_b, ws=ws)
    Ka, Va = synth.decode_tokens(w, layer["Qk"], layer["Qv"], N_APPEND, seed, 0, DEV)
    appends = []
    for s in range(N_APPEND):
        k, v = Ka[:, s:s + 1].contiguous(), Va[:, s:s + 1].contiguous()
        L.lrkv_compress(D, cache, k, v, w.tau, ws=ws)
        appends.append((U.f64(k), U.f64(v)))
    out = U.f64(U.gpu_decode(D, cache, layer["q"], ws))
    torch.cuda.synchronize()
    assert int(cache.dev_status[0]) == 0
    assert cache.seq_len.tolist() == [n + N_APPEND for n in lengths]

    rng = np.random.default_rng(seed)
    picks = {(0, 0), (w.B - 1, w.Hkv - 1),
             (int(rng.integers(w.B)), int(rng.integers(w.Hkv)))}
    U_k, U_v = U.f64(layer["U_k"]), U.f64(layer["U_v"])
    g = w.Hq // w.Hkv
    q = U.f64(layer["q"])
    heads = {}
    for b, h in sorted(picks):
        Kh = U.f64(layer["K"][b:b + 1, :, h:h + 1])
        Vh = U.f64(layer["V"][b:b + 1, :, h:h + 1])
        app_h = [(a[b:b + 1, :, h:h + 1], v[b:b + 1, :, h:h + 1]) for a, v in appends]
        oc, e_ref = _oracle_head(D, U_k[h:h + 1], U_v[h:h + 1], Kh, Vh, w.tau, lengths[b], app_h)
        gc = _gpu_head(D, cache, b, h)
        T = int(oc.seq_len[0])
        assert int(gc.seq_len[0]) == T
        # coefficients of every position: 1 ulp + the fp32 accumulation bound
        X_k = np.concatenate([Kh[0, :lengths[b], 0]] + [a[0, :, 0] for a, _ in app_h])
        X_v = np.concatenate([Vh[0, :lengths[b], 0]] + [v[0, :, 0] for _, v in app_h])
        for got, want, X, Ub in ((gc.coef_k[0, 0, :T], oc.coef_k[0, 0, :T], X_k, U_k[h]),
                                 (gc.coef_v[0, 0, :T], oc.coef_v[0, 0, :T], X_v, U_v[h])):
            tol = O.bf16_ulp(np.maximum(np.abs(got), np.abs(want)))
            tol = tol + U.COEF_ABS_SAFETY * U.GAMMA_128 * (np.abs(X) @ np.abs(Ub))
            bad = np.abs(got - want) > tol
            assert not bad.any(), f"(b={b},h={h}) {bad.sum()} coefficients off the bound"
        # routed sets: identical outside the band around tau
        band = set(np.flatnonzero(np.abs(e_ref - w.tau) < U.BAND).tolist())
        rg, ro = set(U.routed_positions(gc, 0, 0)), set(U.routed_positions(oc, 0, 0))
        assert (rg ^ ro) <= band, f"(b={b},h={h}) routed sets differ: {sorted(rg ^ ro)[:10]}"
        # the list: ascending, matching the mask, rows exact
        n = int(gc.full_cnt[0, 0])
        assert n == len(rg)
        idx = gc.full_idx[0, 0, :n]
        assert np.array_equal(idx, np.array(sorted(rg), dtype=idx.dtype))
        src_k = np.concatenate([Kh[0, :lengths[b], 0]] + [a[0, :, 0] for a, _ in app_h])
        src_v = np.concatenate([Vh[0, :lengths[b], 0]] + [v[0, :, 0] for _, v in app_h])
        assert np.array_equal(gc.full_k[0, 0, :n], src_k[idx])
        assert np.array_equal(gc.full_v[0, 0, :n], src_v[idx])
        # decode over the GPU-written cache
        ref = O.decode_attn(gc, q[b:b + 1, h * g:(h + 1) * g])
        assert U.out_rel_err(out[b, h * g:(h + 1) * g], ref[0]) <= U.OUT_RTOL, (b, h)
        heads[(b, h)] = (oc, band)

    # two fused steps (lrkv_append_decode_attn): the same checks on the sampled heads
    Kf, Vf = synth.decode_tokens(w, layer["Qk"], layer["Qv"], N_APPEND + 2, seed, 0, DEV)
    qf = synth.decode_queries(w, 2, seed + 1, 0, DEV)
    for s in range(2):
        k = Kf[:, N_APPEND + s:N_APPEND + s + 1].contiguous()
        v = Vf[:, N_APPEND + s:N_APPEND + s + 1].contiguous()
        out = torch.empty(w.B, w.Hq, w.d, dtype=torch.float32, device=DEV)
        L.lrkv_append_decode_attn(D, cache, k, v, w.tau, qf[s], out, ws=ws)
        torch.cuda.synchronize()
        assert int(cache.dev_status[0]) == 0
        assert cache.seq_len.tolist() == [n + N_APPEND + s + 1 for n in lengths]
        out = U.f64(out)
        kq, vq, qq = U.f64(k), U.f64(v), U.f64(qf[s])
        for (b, h), (oc, band) in heads.items():
            e1, _, _ = O.compress(oc, kq[b:b + 1, :, h:h + 1], vq[b:b + 1, :, h:h + 1], w.tau)
            gc = _gpu_head(D, cache, b, h)
            T = int(oc.seq_len[0])
            assert int(gc.seq_len[0]) == T
            for got, want, x, Ub in ((gc.coef_k[0, 0, T - 1], oc.coef_k[0, 0, T - 1], kq[b, 0, h], U_k[h]),
                                     (gc.coef_v[0, 0, T - 1], oc.coef_v[0, 0, T - 1], vq[b, 0, h], U_v[h])):
                tol = O.bf16_ulp(np.maximum(np.abs(got), np.abs(want)))
                tol = tol + U.COEF_ABS_SAFETY * U.GAMMA_128 * (np.abs(x) @ np.abs(Ub))
                assert (np.abs(got - want) <= tol).all(), (b, h, s)
            rg, ro = set(U.routed_positions(gc, 0, 0)), set(U.routed_positions(oc, 0, 0))
            assert (rg ^ ro) <= band | ({T - 1} if abs(float(e1.ravel()[0]) - w.tau) < U.BAND else set())
            ref = O.decode_attn(gc, qq[b:b + 1, h * g:(h + 1) * g])
            assert U.out_rel_err(out[b, h * g:(h + 1) * g], ref[0]) <= U.OUT_RTOL, (b, h, s)


def test_long_capacity_holding_8k():
    """A cache allocated for 131072 positions that holds the 8K workload's
    context (the serving case: capacity for the longest request): the decode
    splits follow the live length.  Sampled heads against the oracle, then one
    fused append + decode step."""
    wi, w = 1, synth.workload(1, layers=1)
    seed = 41
    layer = synth.make_layer(w, 0, seed, device=DEV)
    D = U.dims_of(w, 131072, 32768)
    cache = L.LayerCache(D, layer["U_k"], layer["U_v"], device=DEV)
    ws = L.make_workspace(D, DEV)
    L.lrkv_compress(D, cache, layer["K"], layer["V"], w.tau, ws=ws)
    out = U.f64(U.gpu_decode(D, cache, layer["q"], ws))
    Kf, Vf = synth.decode_tokens(w, layer["Qk"], layer["Qv"], 1, seed, 0, DEV)
    o2 = torch.empty(w.B, w.Hq, w.d, dtype=torch.float32, device=DEV)
    # the decode above read the prefilled cache; gather those heads before the fused step
    g = w.Hq // w.Hkv
    q = U.f64(layer["q"])
    torch.cuda.synchronize()
    for h in (0, 5):
        gc = _gpu_head(D, cache, 0, h)
        ref = O.decode_attn(gc, q[0:1, h * g:(h + 1) * g])
        assert U.out_rel_err(out[0, h * g:(h + 1) * g], ref[0]) <= U.OUT_RTOL, h
    L.lrkv_append_decode_attn(D, cache, Kf.contiguous(), Vf.contiguous(), w.tau, layer["q"], o2, ws=ws)
    torch.cuda.synchronize()
    assert int(cache.dev_status[0]) == 0 and int(cache.seq_len[0]) == w.T + 1
    o2 = U.f64(o2)
    for h in (0, 3, 7):
        gc = _gpu_head(D, cache, 0, h)
        ref = O.decode_attn(gc, q[0:1, h * g:(h + 1) * g])
        assert U.out_rel_err(o2[0, h * g:(h + 1) * g], ref[0]) <= U.OUT_RTOL, h


@pytest.mark.parametrize("wi,bits", [(4, 8), (1, 4)], ids=["mha131072_int8", "llama8k_int4"])
def test_full_size_quantised(wi, bits):
    """A quantised cache at full context beside a bf16 cache fed the same calls
    (prefill, one append, one fused append + decode): on sampled heads the codes
    and scales equal the oracle's quantiser applied to the bf16 rows the same
    calls stored (bit for bit), the routing state is the bf16 cache's, and the
    decode matches the oracle's decode over the dequantised rows."""
    w = synth.workload(wi, layers=1)
    seed = 51 + wi
    layer = synth.make_layer(w, 0, seed, device=DEV)
    T_cap = synth.pad_to(w.T + BENCH_EXTRA, 32)
    Db = U.dims_of(w, T_cap, bench_f_cap(wi, T_cap))
    Dq = U.dims_of(w, T_cap, bench_f_cap(wi, T_cap), coef_bits=bits)
    cb = L.LayerCache(Db, layer["U_k"], layer["U_v"], device=DEV)
    cq = L.LayerCache(Dq, layer["U_k"], layer["U_v"], device=DEV)
    wsb, wsq = L.make_workspace(Db, DEV), L.make_workspace(Dq, DEV)
    Ka, Va = synth.decode_tokens(w, layer["Qk"], layer["Qv"], 2, seed, 0, DEV)
    qf = synth.decode_queries(w, 1, seed, 0, DEV)
    outs = []
    for D, c, ws in ((Db, cb, wsb), (Dq, cq, wsq)):
        L.lrkv_compress(D, c, layer["K"], layer["V"], w.tau, ws=ws)
        L.lrkv_compress(D, c, Ka[:, :1].contiguous(), Va[:, :1].contiguous(), w.tau, ws=ws)
        o = torch.empty(w.B, w.Hq, w.d, dtype=torch.float32, device=DEV)
        L.lrkv_append_decode_attn(D, c, Ka[:, 1:2].contiguous(), Va[:, 1:2].contiguous(), w.tau, qf[0], o, ws=ws)
        outs.append(o)
    torch.cuda.synchronize()
    assert int(cq.dev_status[0]) == 0 and int(cb.dev_status[0]) == 0
    for f in ("route_mask", "full_idx", "full_cnt", "seq_len"):
        assert torch.equal(getattr(cq, f), getattr(cb, f)), f
    out = U.f64(outs[1])
    q = U.f64(qf[0])
    g = w.Hq // w.Hkv
    T = int(cq.seq_len[0])
    rng = np.random.default_rng(seed)
    for h in sorted({0, w.Hkv - 1, int(rng.integers(w.Hkv))}):
        gb = _gpu_head(Db, cb, 0, h)
        want = O.quantize_cache(gb, bits)
        codes = lambda t: t.cpu().numpy().view(np.int8) if bits == 8 else O.unpack_int4(t.cpu().numpy())
        qk, qv = codes(cq.coef_k[0, h, :T]), codes(cq.coef_v[0, h, :T])
        sk, sv = cq.scale_k[0, h, :T].cpu().numpy(), cq.scale_v[0, h, :T].cpu().numpy()
        assert np.array_equal(qk, want["qk"][0, 0, :T]) and np.array_equal(sk, want["sk"][0, 0, :T]), h
        assert np.array_equal(qv, want["qv"][0, 0, :T]) and np.array_equal(sv, want["sv"][0, 0, :T]), h
        gq = gb
        gq.coef_k[0, 0, :T] = O.dequantize_coef(qk, sk)
        gq.coef_v[0, 0, :T] = O.dequantize_coef(qv, sv)
        ref = O.decode_attn(gq, q[0:1, h * g:(h + 1) * g])
        assert U.out_rel_err(out[0, h * g:(h + 1) * g], ref[0]) <= U.OUT_RTOL, h


def test_full_size_attention_aware():
    """The 8K workload with an attention-aware key basis (Theorem 1 from seeded
    calibration queries and the head's keys): sampled heads' coefficients,
    routing and decode against the oracle's aware cache."""
    from tests.test_gpu_aware import _aware_bases
    w = synth.workload(1, layers=1)
    seed = 57
    layer = synth.make_layer(w, 0, seed, device=DEV)
    T_cap = synth.pad_to(w.T + BENCH_EXTRA, 32)
    # the aware key basis routes far more than the orthonormal one here (its
    # mean is not in the span): a list for every position
    D = U.dims_of(w, T_cap, T_cap)
    K64 = U.f64(layer["K"])
    Wk, Wq, mu = _aware_bases(K64, w.r_k, seed)
    t = lambda a, dt: torch.from_numpy(a).to(dt).to(DEV)
    cache = L.LayerCache(D, t(Wk, torch.bfloat16), layer["U_v"], device=DEV,
                         U_kq=t(Wq, torch.bfloat16), mu_k=t(mu, torch.float32))
    ws = L.make_workspace(D, DEV)
    L.lrkv_compress(D, cache, layer["K"], layer["V"], w.tau, ws=ws)
    Ka, Va = synth.decode_tokens(w, layer["Qk"], layer["Qv"], 1, seed, 0, DEV)
    o = torch.empty(w.B, w.Hq, w.d, dtype=torch.float32, device=DEV)
    L.lrkv_append_decode_attn(D, cache, Ka.contiguous(), Va.contiguous(), w.tau, layer["q"], o, ws=ws)
    torch.cuda.synchronize()
    assert int(cache.dev_status[0]) == 0
    out, q = U.f64(o), U.f64(layer["q"])
    g = w.Hq // w.Hkv
    V64, Uv = U.f64(layer["V"]), U.f64(layer["U_v"])
    for h in (0, 3, 7):
        od = O.Dims(B=1, Hq=g, Hkv=1, d=w.d, r_k=w.r_k, r_v=w.r_v, T_cap=T_cap, F_cap=D.F_cap)
        oc = O.Cache.empty(od, Wk[h:h + 1], Uv[h:h + 1], U_kq=Wq[h:h + 1], mu_k=mu[h:h + 1])
        e0, _, _ = O.compress(oc, K64[:, :, h:h + 1], V64[:, :, h:h + 1], w.tau)
        e1, _, _ = O.compress(oc, U.f64(Ka)[:, :, h:h + 1], U.f64(Va)[:, :, h:h + 1], w.tau)
        e_ref = np.concatenate([e0[0, 0], e1[0, 0]])
        gc = _gpu_head(D, cache, 0, h)
        gc.U_kq, gc.mu_k = oc.U_kq, oc.mu_k
        T = int(oc.seq_len[0])
        X = np.concatenate([K64[0, :, h], U.f64(Ka)[0, :, h]])
        tol = O.bf16_ulp(np.maximum(np.abs(gc.coef_k[0, 0, :T]), np.abs(oc.coef_k[0, 0, :T])))
        tol = tol + U.COEF_ABS_SAFETY * U.GAMMA_128 * ((np.abs(X) + np.abs(mu[h])) @ np.abs(Wk[h]))
        assert (np.abs(gc.coef_k[0, 0, :T] - oc.coef_k[0, 0, :T]) <= tol).all(), h
        band = set(np.flatnonzero(np.abs(e_ref - w.tau) < U.BAND).tolist())
        rg, ro = set(U.routed_positions(gc, 0, 0)), set(U.routed_positions(oc, 0, 0))
        assert (rg ^ ro) <= band, h
        ref = O.decode_attn(gc, q[0:1, h * g:(h + 1) * g])
        assert U.out_rel_err(out[0, h * g:(h + 1) * g], ref[0]) <= U.OUT_RTOL, h
