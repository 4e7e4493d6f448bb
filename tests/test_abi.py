"""The C ABI without a GPU: the library loads, exports every symbol that
include/lrkv.h declares, sizes workspaces, and rejects bad arguments on the
host before anything is launched."""
import ctypes
import os
import re
import subprocess

import pytest

import decode_attention_lrkv_b200 as L
from decode_attention_lrkv_b200 import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "lrkv.h")


@pytest.fixture(scope="module")
def lib():
    build.build()
    return L.load_library()


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(lrkv_[a-z_0-9]+)\s*\(", src)))


def test_header_declares_the_boundary():
    assert declared_functions() == sorted(
        ["lrkv_workspace_size", "lrkv_compress", "lrkv_decode_attn", "lrkv_decode_attn_noalloc",
         "lrkv_append_decode_attn", "lrkv_fit_workspace_size", "lrkv_fit_basis",
         "lrkv_rank_for_budget", "lrkv_status_str", "lrkv_oja_workspace_size", "lrkv_oja_update"])


def test_every_declared_symbol_is_exported(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name
    out = subprocess.run(["nm", "-D", "--defined-only", L.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\bT (lrkv_\w+)", out))
    assert set(declared_functions()) <= exported
    # nothing but the declared C ABI is exported
    assert exported == set(declared_functions())


def test_status_strings(lib):
    for code in range(5):
        assert L.lrkv_status_str(code)
    assert L.lrkv_status_str(0) == "ok"
    assert "unknown" in L.lrkv_status_str(99)


def _dims(**kw):
    base = dict(B=2, Hq=32, Hkv=8, d=128, r_k=64, r_v=96, T_cap=8192, F_cap=1024)
    base.update(kw)
    return L.Dims(**base)


def test_workspace_size(lib):
    n = L.lrkv_workspace_size(_dims())
    assert n > 0 and n % 256 == 0
    assert L.lrkv_workspace_size(_dims(T_cap=16384)) > n
    assert L.lrkv_workspace_size(_dims(coef_bits=8)) == n       # the format needs no workspace
    for bad in (dict(d=64), dict(r_k=40), dict(r_v=0), dict(r_k=144), dict(Hq=30),
                dict(T_cap=100), dict(T_cap=0), dict(F_cap=-1), dict(B=0), dict(Hq=72, Hkv=8),
                dict(coef_bits=3), dict(coef_bits=32)):
        assert L.lrkv_workspace_size(_dims(**bad)) == 0, bad
    assert lib.lrkv_workspace_size(None) == 0


class _FakeCache:
    """Cache-shaped object with fake, never-dereferenced device addresses."""
    def __init__(self, base=0x10000000, **override):
        self.ptrs = {f: base + 0x1000000 * i for i, f in enumerate(L.LayerCache.FIELDS)}
        self.ptrs.update(override)

    def c(self):
        return L._Cache(*[self.ptrs[f] for f in L.LayerCache.FIELDS])


def _call_compress(lib, dims, cache, k=0x20000000, v=0x30000000, t_new=4, t_new_b=None,
                   err=None, ws=0x40000000, ws_bytes=None):
    if ws_bytes is None:
        ws_bytes = lib.lrkv_workspace_size(ctypes.byref(dims.c())) if dims else 1 << 30
    return lib.lrkv_compress(ctypes.byref(dims.c()) if dims else None,
                             ctypes.byref(cache.c()) if cache else None, k, v, t_new, t_new_b,
                             0.25, err, ws, ws_bytes, None)


def _call_decode(lib, dims, cache, q=0x20000000, out=0x30000000, ws=0x40000000, ws_bytes=None):
    if ws_bytes is None:
        ws_bytes = lib.lrkv_workspace_size(ctypes.byref(dims.c())) if dims else 1 << 30
    return lib.lrkv_decode_attn(ctypes.byref(dims.c()) if dims else None,
                                ctypes.byref(cache.c()) if cache else None, q, out, ws, ws_bytes,
                                None)


def _decode_records(D):
    """Split records per (b, kv head) in lrkv_workspace_size(D): the decode's
    region comes last, after the decode tickets, the compress ticket, the row
    tickets, the prefill's per-token errors and its per-tile counts and bits
    (each region rounded up to 256 bytes), and holds
    [B][Hkv][records][g][4 + r_v + d] fp32, g raised to 4 for groups of 3."""
    a = lambda x: (x + 255) // 256 * 256
    bh = D.B * D.Hkv
    n_tiles = (D.T_cap + 127) // 128
    fixed = a(4 * bh) + a(4) + a(4 * D.B) + a(8 * bh * D.T_cap) + a(4 * bh * n_tiles) + a(16 * bh * n_tiles)
    g = D.Hq // D.Hkv
    g = 4 if 2 < g < 4 else g
    return (L.lrkv_workspace_size(D) - fixed) // (4 * bh * g * (4 + D.r_v + D.d))


def test_decode_records_hold_the_fewest_splits_and_the_append(lib):
    """A fused append + decode streams the cached positions over at most
    records - 1 splits of at most 8192 positions (its grid's last CTA appends),
    so for any cached length up to T_cap the workspace must hold
    ceil(T_cap / 8192) + 1 records per (b, kv head).  The cases include T_cap
    just past a multiple of 8192 with many (b, kv head) pairs, where the split
    model gives a full cache exactly ceil(T_cap / 8192) splits (no SMs are
    visible here: the model assumes 148)."""
    for B, Hkv in ((1, 1), (1, 8), (2, 8), (8, 8), (16, 8), (1, 32), (64, 8)):
        for T_cap in (32, 8192, 8224, 16416, 24608, 65568, 131136, 139296):
            D = _dims(B=B, Hkv=Hkv, Hq=4 * Hkv, T_cap=T_cap, F_cap=32)
            assert _decode_records(D) >= -(-T_cap // 8192) + 1, (B, Hkv, T_cap)
    # the shape that needs the extra record: the model gives 8224 positions two splits
    assert _decode_records(_dims(B=8, Hkv=8, Hq=32, T_cap=8224, F_cap=32)) == 3


def test_host_validation_rejects_before_launch(lib):
    D = _dims()
    C = _FakeCache()
    INVALID, UNSUP, ALIGN = 1, 2, 3
    assert _call_compress(lib, None, C) == INVALID
    assert _call_compress(lib, D, None) == INVALID
    assert _call_compress(lib, _dims(d=64), C, ws_bytes=1 << 30) == UNSUP
    assert _call_compress(lib, _dims(Hq=33), C, ws_bytes=1 << 30) == INVALID
    assert _call_compress(lib, D, C, k=None) == INVALID
    assert _call_compress(lib, D, C, t_new=-1) == INVALID
    assert _call_compress(lib, D, _FakeCache(seq_len=None)) == INVALID
    assert _call_compress(lib, D, _FakeCache(coef_k=0x10000008)) == ALIGN
    assert _call_compress(lib, D, C, v=0x30000004) == ALIGN
    assert _call_compress(lib, D, C, t_new_b=0x50000002) == ALIGN
    assert _call_compress(lib, D, C, ws=None) == INVALID
    assert _call_compress(lib, D, C, ws_bytes=16) == INVALID
    assert _call_compress(lib, D, C, ws=0x40000001) == ALIGN
    assert _call_compress(lib, D, C, t_new=0) == 0          # nothing to append: no launch
    assert _call_decode(lib, None, C) == INVALID
    assert _call_decode(lib, D, C, q=None) == INVALID
    assert _call_decode(lib, D, C, out=0x30000002) == ALIGN
    assert _call_decode(lib, D, C, ws_bytes=1) == INVALID
    assert _call_decode(lib, _dims(Hq=72), C, ws_bytes=1 << 30) == UNSUP
    # F_cap = 0 lets the full-rank buffers be null; otherwise they are required
    assert _call_compress(lib, _dims(F_cap=0), _FakeCache(full_k=None, full_v=None, full_idx=None),
                          t_new=0) == 0
    assert _call_compress(lib, D, _FakeCache(full_v=None)) == INVALID
    # quantised coefficients need their per-row scales
    Dq = _dims(coef_bits=8)
    assert _call_compress(lib, Dq, _FakeCache(scale_v=None)) == INVALID
    assert _call_decode(lib, Dq, _FakeCache(scale_k=0x50000008)) == ALIGN
    assert _call_compress(lib, D, _FakeCache(scale_k=None, scale_v=None), t_new=0) == 0   # bf16: unused
    # the attention-aware key basis and mean are optional, aligned when given
    assert _call_compress(lib, D, _FakeCache(U_kq=None, mu_k=None), t_new=0) == 0
    assert _call_compress(lib, D, _FakeCache(mu_k=0x50000004)) == ALIGN
    assert _call_decode(lib, D, _FakeCache(U_kq=0x50000002)) == ALIGN


def test_rank_for_budget_matches_the_oracle(lib):
    """Host call: the same rank as the oracle on fp32 spectra, bit for bit, including
    budgets that land exactly on a discarded-mass boundary."""
    import numpy as np
    import torch
    import oracle as O
    rng = np.random.default_rng(11)
    spectra = [np.sort(rng.gamma(a, 1.0, 128).astype(np.float32))[::-1] for a in (0.3, 1.0, 3.0)]
    spectra.append(np.array([2.0 ** -j for j in range(128)], np.float32))   # exact binary fractions
    z = np.zeros(128, np.float32)
    z[:3] = [5.0, 2.0, 1.0]
    z[-1] = -1e-6                                                             # rounding below zero
    spectra.append(z)
    spectra.append(np.zeros(128, np.float32))
    lam = np.stack(spectra)
    for budget in (0.0, 1e-6, 0.01, 0.075, 0.125, 0.25, 0.5, 1.0, 0.5 ** 10):
        got = L.lrkv_rank_for_budget(torch.from_numpy(lam.copy()), budget)
        want = [O.rank_for_budget(row, budget) for row in lam]
        assert got.tolist() == want, budget


def test_rank_for_budget_rejects_bad_arguments(lib):
    import ctypes
    import numpy as np
    lam = np.ones((2, 8), np.float32)
    r = np.full(2, -7, np.int32)
    P = lambda a: a.ctypes.data
    bad = L.LRKV_ERR_INVALID_ARG
    assert lib.lrkv_rank_for_budget(None, 2, 8, 0.1, P(r)) == bad
    assert lib.lrkv_rank_for_budget(P(lam), 2, 8, 0.1, None) == bad
    assert lib.lrkv_rank_for_budget(P(lam), 0, 8, 0.1, P(r)) == bad
    assert lib.lrkv_rank_for_budget(P(lam), 2, 0, 0.1, P(r)) == bad
    assert lib.lrkv_rank_for_budget(P(lam), 2, 4097, 0.1, P(r)) == bad
    for b in (-0.01, 1.01, float("nan")):
        assert lib.lrkv_rank_for_budget(P(lam), 2, 8, b, P(r)) == bad
    assert (r == -7).all()
    assert lib.lrkv_rank_for_budget(P(lam), 2, 8, 0.5, P(r)) == L.LRKV_OK
    assert r.tolist() == [4, 4]


def test_oja_update_rejects_bad_arguments(lib):
    D = _dims()
    INVALID, UNSUP, ALIGN = 1, 2, 3
    n = L.lrkv_oja_workspace_size(D, 1000, 64)
    assert n > 0 and L.lrkv_oja_workspace_size(D, 1000, 40) == 0 and L.lrkv_oja_workspace_size(D, 0, 64) == 0
    call = lambda dims=D, X=0x20000000, n_rows=1000, r=64, eta=0.1, U=0x30000000, U_out=None, \
        ws=0x40000000, ws_bytes=n: lib.lrkv_oja_update(ctypes.byref(dims.c()), X, n_rows, r, eta, U, U_out,
                                                       ws, ws_bytes, None)
    assert call(X=None) == INVALID and call(U=None) == INVALID and call(r=8) == INVALID
    assert call(r=144) == INVALID and call(n_rows=0) == INVALID
    assert call(eta=-0.5) == INVALID and call(eta=float("nan")) == INVALID and call(eta=float("inf")) == INVALID
    assert call(dims=_dims(d=64)) == UNSUP
    assert call(X=0x20000008) == ALIGN and call(U_out=0x50000004) == ALIGN
    assert call(ws_bytes=n - 1) == INVALID and call(ws=None) == INVALID
