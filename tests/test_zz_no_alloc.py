"""sa_forward_noalloc: the SA forward for callers that cannot allocate device memory.

Callers such as plugins that only receive input and output pointers, or code running inside a
memory pool it does not own, cannot create a workspace. sa_forward_noalloc serves them from a
fixed device array inside libska.so. These tests call it through the C ABI and check that two
calls in a row give bit for bit the sketch and lse of sa_forward with a caller-provided workspace
(the same kernels on the same schedule), for both normalisations and for fp32 inputs (whose bf16
copies also live in the array), that a problem larger than the array is refused before anything
runs, and that a device-side error of a call can be read back through
sa_forward_noalloc_read_status.

The file is named so that pytest collects it last.
"""
import ctypes

import numpy as np
import pytest
import torch

from sketch_attention_flashsa_b200 import _lib
from sketch_attention_flashsa_b200 import workloads as W

pytestmark = pytest.mark.gpu

def _p(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else ctypes.c_void_p(0)


def _desc(inp, norm="proto"):
    from sketch_attention_flashsa_b200 import api
    return api.sa_desc(inp.q, inp.k, inp.cu_seqlens, scale=inp.scale, norm=norm)


def _run(inp, noalloc: bool, norm="proto"):
    L = _lib.lib()
    dev = "cuda"
    q, k, v, cu = (x.to(dev) for x in (inp.q, inp.k, inp.v, inp.cu_seqlens))
    su = inp.seqused.to(dev) if inp.seqused is not None else None
    d = _desc(inp, norm)
    sk = torch.empty((d.num_users, d.num_heads, d.num_protos, d.head_dim), dtype=torch.float32, device=dev)
    lse_shape = (d.total_tokens, d.num_heads) if norm == "proto" else (d.num_users, d.num_heads, d.num_protos)
    lse = torch.empty(lse_shape, dtype=torch.float32, device=dev)
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


def _same(got, want):
    """Bit for bit (NaN-free outputs; -inf lse entries compare equal)."""
    assert got.shape == want.shape
    assert np.array_equal(got, want)


CASES = {
    "proto_d128_k512_padded": (lambda: W.make_sa([700, 0, 129, 300], 2, 128, 512, seed=201,
                                                 seqused=[650, 0, 129, 300]), "proto"),
    "proto_d64_k256": (lambda: W.make_sa([1000, 77], 4, 64, 256, seed=202), "proto"),
    "token_d128_k384": (lambda: W.make_sa([900, 5, 300], 2, 128, 384, seed=203, norm=W.NORM_TOKEN), "token"),
    "proto_fp32_config1": (W.config1, "proto"),
    "token_fp32_config1": (W.config1, "token"),
}


@pytest.mark.parametrize("name", sorted(CASES))
def test_noalloc_matches_workspace_entry_point_twice(name):
    make, norm = CASES[name]
    inp = make()
    want_sk, want_lse = _run(inp, noalloc=False, norm=norm)
    for _ in range(2):  # the array keeps the previous call's contents: nothing may carry over
        got_sk, got_lse = _run(inp, noalloc=True, norm=norm)
        _same(got_sk, want_sk)
        _same(got_lse, want_lse)


def test_noalloc_reports_device_errors():
    """A bounded wait made to run out (debug flag 1 withholds one producer arrival) is recorded in
    the array's status word and read back through sa_forward_noalloc_read_status; the next call is
    correct again."""
    from sketch_attention_flashsa_b200 import api
    L = _lib.lib()
    inp = W.make_sa([600, 300], 2, 128, 512, seed=204)
    want_sk, want_lse = _run(inp, noalloc=False)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    assert L.sa_forward_noalloc_read_status(stream) == _lib.SKA_OK
    try:
        api.set_debug(50_000_000, 1)
        _run(inp, noalloc=True)
    finally:
        api.set_debug(0, 0)
    assert L.sa_forward_noalloc_read_status(stream) == _lib.SKA_ERR_DEVICE_TIMEOUT
    assert L.sa_forward_noalloc_read_status(stream) == _lib.SKA_OK  # read clears it
    got_sk, got_lse = _run(inp, noalloc=True)
    _same(got_sk, want_sk)
    _same(got_lse, want_lse)


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
