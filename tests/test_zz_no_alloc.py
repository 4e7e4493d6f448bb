"""lrkv_decode_attn_noalloc: decode attention for callers that cannot allocate.

Some callers may not allocate device memory on the decode path (an inference
engine's plugin hook that only gets memory at build time, a latency-critical
loop where cudaMalloc's cost and device synchronisation are unacceptable, a C
caller without a device allocator).  This entry point takes its split-K
scratch from a device array the library holds instead of a workspace.  Its
output must match lrkv_decode_attn's, within the parity tolerance, call
after call: the shared array keeps the previous call's contents, so each
call has to start from cleared tickets.  Shapes of both decode kernels are
covered (the streaming kernel at GQA 4 and 3; the CUDA-core kernel, ranks
32/48), and one call is checked against the fp64 oracle as well.  This file is
collected last.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle as O
import synth
import decode_attention_lrkv_b200 as L
from tests import lrkv_testutil as U

pytestmark = pytest.mark.gpu

OUT_RTOL = 2e-3     # the parity bar used for every decode output


def _rel(a, b):
    a, b = a.double().cpu().numpy(), b.double().cpu().numpy()
    return np.abs(a - b).max() / max(np.abs(b).max(), 1e-30)


def _noalloc(lib, D, cache, q, out, stream):
    return lib.lrkv_decode_attn_noalloc(ctypes.byref(D.c()), ctypes.byref(cache.c()),
                                        ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(out.data_ptr()),
                                        ctypes.c_void_p(stream.cuda_stream))


@pytest.mark.parametrize("Hq,r_k,r_v", [(32, 64, 96), (24, 64, 96), (24, 32, 48)],
                         ids=["gqa4_streaming", "gqa3_streaming", "gqa3_cuda_cores"])
def test_noalloc_matches_workspace_decode_on_consecutive_calls(Hq, r_k, r_v):
    dev = torch.device("cuda", 0)
    w = synth.workload(1, Hq=Hq, r_k=r_k, r_v=r_v, T=3000, layers=1)
    lay = synth.make_layer(w, 0, 77, device=dev)
    D = L.Dims(B=w.B, Hq=w.Hq, Hkv=w.Hkv, d=w.d, r_k=w.r_k, r_v=w.r_v, T_cap=3008, F_cap=3008)
    cache = L.LayerCache(D, lay["U_k"], lay["U_v"], device=dev)
    ws = L.make_workspace(D, dev)
    L.lrkv_compress(D, cache, lay["K"], lay["V"], w.tau, ws=ws)
    qs = synth.decode_queries(w, 2, 77, 0, dev)
    lib = L.load_library()
    stream = torch.cuda.current_stream()
    for i in range(2):                       # two calls in a row share the library's scratch
        ref = torch.empty(w.B, w.Hq, w.d, dtype=torch.float32, device=dev)
        L.lrkv_decode_attn(D, cache, qs[i], ref, ws=ws)
        out = torch.full((w.B, w.Hq, w.d), float("nan"), dtype=torch.float32, device=dev)
        code = _noalloc(lib, D, cache, qs[i], out, stream)
        assert code == L.LRKV_OK, L.lrkv_status_str(code)
        torch.cuda.synchronize()
        assert torch.isfinite(out).all()
        assert _rel(out, ref) <= OUT_RTOL
        if i == 1:                           # and against the oracle on the GPU-written cache
            gc = U.gpu_to_oracle(D, cache)
            assert U.out_rel_err(U.f64(out), O.decode_attn(gc, U.f64(qs[i]))) <= OUT_RTOL


def test_noalloc_rejects_sizes_beyond_its_scratch():
    """Sizes whose split-K scratch exceeds the library's array are refused before
    any pointer is looked at (null pointers here), so nothing is launched."""
    dev = torch.device("cuda", 0)
    big = L.Dims(B=64, Hq=64, Hkv=8, d=128, r_k=64, r_v=96, T_cap=65536, F_cap=32)
    null_cache = L._Cache(*([None] * len(L.LayerCache.FIELDS)))
    lib = L.load_library()
    code = lib.lrkv_decode_attn_noalloc(ctypes.byref(big.c()), ctypes.byref(null_cache), None, None,
                                        ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream))
    assert code == 2          # LRKV_ERR_UNSUPPORTED: needs more than LRKV_NOALLOC_SCRATCH_BYTES
    # sizes that fit, with the same null pointers: the pointer check refuses them
    small = L.Dims(B=1, Hq=32, Hkv=8, d=128, r_k=64, r_v=96, T_cap=4096, F_cap=32)
    code = lib.lrkv_decode_attn_noalloc(ctypes.byref(small.c()), ctypes.byref(null_cache), None, None,
                                        ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream))
    assert code == L.LRKV_ERR_INVALID_ARG
