"""sa_forward_noalloc: the SA forward for callers that cannot allocate device memory.

Callers such as plugins that only receive input and output pointers, or code running inside a
memory pool it does not own, cannot create a workspace. sa_forward_noalloc serves them from a
fixed device array inside libska.so. These tests call it through the C ABI and check that two
calls in a row give the same sketch and lse as sa_forward with a caller-provided workspace,
within the parity tolerance of the other GPU tests, and that a problem larger than the array
is refused before anything runs.

The file is named so that pytest collects it last.
"""
import ctypes

import numpy as np
import pytest
import torch

from sketch_attention_flashsa_b200 import _lib
from sketch_attention_flashsa_b200 import workloads as W

pytestmark = pytest.mark.gpu

MAX_ABS = 1e-2
REL_L2 = 5e-3


def _p(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else ctypes.c_void_p(0)


def _desc(inp):
    from sketch_attention_flashsa_b200 import api
    return api.sa_desc(inp.q, inp.k, inp.cu_seqlens, scale=inp.scale, norm="proto")


def _run(inp, noalloc: bool):
    L = _lib.lib()
    dev = "cuda"
    q, k, v, cu = (x.to(dev) for x in (inp.q, inp.k, inp.v, inp.cu_seqlens))
    su = inp.seqused.to(dev) if inp.seqused is not None else None
    d = _desc(inp)
    sk = torch.empty((d.num_users, d.num_heads, d.num_protos, d.head_dim), dtype=torch.float32, device=dev)
    lse = torch.empty((d.total_tokens, d.num_heads), dtype=torch.float32, device=dev)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    if noalloc:
        rc = L.sa_forward_noalloc(ctypes.byref(d), _p(q), _p(k), _p(v), _p(cu), _p(su), _p(sk), _p(lse), None,
                                  stream)
    else:
        ws = torch.empty(L.sa_forward_workspace_size(ctypes.byref(d)), dtype=torch.uint8, device=dev)
        rc = L.sa_forward(ctypes.byref(d), _p(q), _p(k), _p(v), _p(cu), _p(su), _p(sk), _p(lse), None, _p(ws),
                          ctypes.c_size_t(ws.numel()), stream)
    assert rc == 0, _lib.status_string(rc)
    torch.cuda.synchronize()
    return sk.cpu().numpy().astype(np.float64), lse.cpu().numpy().astype(np.float64)


def _close(got, want):
    fin = np.isfinite(want)
    assert (np.isfinite(got) == fin).all()
    err = np.abs(got[fin] - want[fin])
    assert err.max() <= MAX_ABS
    assert np.linalg.norm(got[fin] - want[fin]) <= REL_L2 * max(np.linalg.norm(want[fin]), 1e-30)


def test_noalloc_matches_workspace_entry_point_twice():
    first = W.make_sa([700, 0, 129, 300], 2, 128, 512, seed=201, seqused=[650, 0, 129, 300])
    second = W.make_sa([1000, 77], 4, 64, 256, seed=202)
    for inp in (first, second):
        want_sk, want_lse = _run(inp, noalloc=False)
        got_sk, got_lse = _run(inp, noalloc=True)
        _close(got_sk, want_sk)
        _close(got_lse, want_lse)


def test_noalloc_refuses_problems_beyond_its_scratch():
    L = _lib.lib()
    cap = L.sa_forward_noalloc_scratch_bytes()
    d = _lib.SaDesc()
    d.num_users, d.num_heads, d.head_dim, d.num_protos = 4096, 16, 128, 512
    d.total_tokens, d.scale = 4096 * 16, 1.0
    assert L.sa_forward_workspace_size(ctypes.byref(d)) > cap
    # refused on the host before any pointer is used or anything is launched
    rc = L.sa_forward_noalloc(ctypes.byref(d), None, None, None, None, None, None, None, None,
                              ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == _lib.SKA_ERR_WORKSPACE_TOO_SMALL
