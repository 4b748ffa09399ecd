"""The C ABI without a GPU: libska.so loads, exports exactly the calls the header declares, and
rejects bad arguments on the host before it touches a device (the header's error contract:
invalid arguments are reported before anything is launched). Fake, never-dereferenced
addresses stand in for device pointers."""
import ctypes
import os
import re
import subprocess

import pytest

from sketch_attention_flashsa_b200 import _lib as L

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "sketch_attn.h")

A = 1 << 32  # a fake address: multiples of it are 256-byte aligned and 4 GiB apart, so no
#               two fake buffers overlap


def header_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return set(re.findall(r"^SKA_API\s+[\w\s\*]*?\b(\w+)\s*\(", text, flags=re.M))


def exported_symbols():
    out = subprocess.run(["nm", "-D", "--defined-only", L.LIB_PATH], capture_output=True, text=True, check=True)
    return {ln.split()[-1] for ln in out.stdout.splitlines() if len(ln.split()) == 3 and ln.split()[1] == "T"}


def test_header_declares_the_boundary():
    names = header_functions()
    assert {"sa_forward", "sa_backward", "stca_forward", "sa_forward_workspace_size",
            "sa_backward_workspace_size", "stca_forward_workspace_size", "ska_status_string"} <= names


def test_library_loads_and_exports_every_declared_call():
    lib = L.lib()
    names = header_functions()
    for n in names:
        assert hasattr(lib, n), n
    assert exported_symbols() == names, "libska.so exports exactly the header's calls"
    assert set(L.EXPORTED) == names, "the binding wraps every declared call"


def test_status_strings():
    want = {L.SKA_OK: "SKA_OK", L.SKA_ERR_INVALID_VALUE: "SKA_ERR_INVALID_VALUE",
            L.SKA_ERR_UNSUPPORTED: "SKA_ERR_UNSUPPORTED", L.SKA_ERR_WORKSPACE_TOO_SMALL: "SKA_ERR_WORKSPACE_TOO_SMALL",
            L.SKA_ERR_CUDA: "SKA_ERR_CUDA", L.SKA_ERR_DEVICE_TIMEOUT: "SKA_ERR_DEVICE_TIMEOUT",
            L.SKA_ERR_RANGE: "SKA_ERR_RANGE"}
    for code, name in want.items():
        assert L.status_string(code) == name
    assert L.status_string(99) not in want.values()


def sa_desc(**kw):
    f = dict(num_users=2, num_heads=2, head_dim=64, num_protos=256, total_tokens=1000, max_seqlen=600, scale=1.0,
             norm=L.SKA_NORM_PROTO, in_dtype=L.SKA_BF16, q_per_user=0, reserved=0)
    f.update(kw)
    return L.SaDesc(*[f[n] for n, _ in L.SaDesc._fields_])


def stca_desc(**kw):
    f = dict(num_users=2, num_heads=2, head_dim=64, num_sketch=256, total_targets=100, total_hist=1000,
             max_targets=60, max_hist=600, scale=0.125, reserved=0)
    f.update(kw)
    return L.StcaDesc(*[f[n] for n, _ in L.StcaDesc._fields_])


def fwd(desc, q=A, k=2 * A, v=3 * A, cu=4 * A, su=None, sk=5 * A, lse=6 * A, mass=None, ws=256 * A,
        ws_bytes=1 << 30):
    return L.lib().sa_forward(ctypes.byref(desc) if desc is not None else None, q, k, v, cu, su, sk, lse, mass, ws,
                              ws_bytes, None)


def bwd(desc, q=A, k=2 * A, v=3 * A, cu=4 * A, su=None, sk=5 * A, lse=6 * A, dsk=7 * A, dq=8 * A, dk=9 * A,
        dv=10 * A, ws=256 * A, ws_bytes=1 << 30):
    return L.lib().sa_backward(ctypes.byref(desc) if desc is not None else None, q, k, v, cu, su, sk, lse, dsk, dq,
                               dk, dv, ws, ws_bytes, None)


def stca(desc, q=A, cut=2 * A, kh=3 * A, vh=4 * A, cuh=5 * A, kvl=None, ks=6 * A, vs=7 * A, out=8 * A, lse=9 * A,
         ws=256 * A, ws_bytes=1 << 30):
    return L.lib().stca_forward(ctypes.byref(desc) if desc is not None else None, q, cut, kh, vh, cuh, kvl, ks, vs,
                                out, lse, ws, ws_bytes, None)


INVALID, UNSUP = L.SKA_ERR_INVALID_VALUE, L.SKA_ERR_UNSUPPORTED


@pytest.mark.parametrize("kw,code", [
    ({"num_heads": 0}, INVALID), ({"num_users": -1}, INVALID), ({"total_tokens": -5}, INVALID),
    ({"total_tokens": 1 << 31}, INVALID), ({"scale": 0.0}, INVALID), ({"scale": -1.0}, INVALID),
    ({"scale": float("nan")}, INVALID), ({"scale": float("inf")}, INVALID), ({"norm": 7}, INVALID),
    ({"in_dtype": 5}, INVALID), ({"q_per_user": 2}, INVALID), ({"num_protos": 0}, INVALID),
    ({"head_dim": 96}, UNSUP), ({"head_dim": 256}, UNSUP),
    # the tile stream H * (T / 128 + B) must stay below 2^31 (32-bit tile indices on the device)
    ({"num_heads": 1 << 16, "total_tokens": (1 << 31) - 1}, INVALID),
])
def test_sa_forward_rejects_bad_descriptors(kw, code):
    assert fwd(sa_desc(**kw)) == code


def test_sa_forward_pointer_checks():
    d = sa_desc()
    assert fwd(None) == INVALID
    assert fwd(d, mass=11 * A + 4) == INVALID  # 16-byte alignment of the mass output
    assert fwd(d, mass=5 * A) == INVALID  # the mass output may not overlap the sketch
    assert fwd(d, q=None) == INVALID
    assert fwd(d, k=None) == INVALID
    assert fwd(d, sk=None) == INVALID
    assert fwd(d, cu=None) == INVALID
    assert fwd(d, ws=None) == INVALID
    assert fwd(d, q=A + 8) == INVALID  # 16-byte alignment
    assert fwd(d, ws=256 * A + 128) == INVALID  # 256-byte workspace alignment
    assert fwd(d, cu=4 * A + 2) == INVALID


def test_empty_batch_is_a_no_op_on_the_host():
    # nothing to do: the call returns before any pointer or device check
    assert fwd(sa_desc(num_users=0, total_tokens=0), q=None, k=None, v=None, cu=None, sk=None, ws=None) == L.SKA_OK
    assert stca(stca_desc(total_targets=0), q=None, out=None, ws=None) == L.SKA_OK


@pytest.mark.parametrize("kw,code", [
    ({"in_dtype": L.SKA_F32}, UNSUP), ({"num_protos": 48}, UNSUP),
    # beyond one CTA: multiples of the chunk (256 at d = 64, 128 at d = 128) up to 4096 only
    ({"num_protos": 640}, UNSUP), ({"num_protos": 8192}, UNSUP), ({"head_dim": 128, "num_protos": 200}, UNSUP),
    ({"head_dim": 128, "num_protos": 4224}, UNSUP), ({"scale": 0.0}, INVALID), ({"norm": 3}, INVALID),
])
def test_sa_backward_rejects(kw, code):
    assert bwd(sa_desc(**kw)) == code


@pytest.mark.parametrize("kw", [{"num_protos": 512}, {"num_protos": 4096}, {"head_dim": 128, "num_protos": 256},
                                {"head_dim": 128, "num_protos": 384}, {"head_dim": 128, "num_protos": 1024}])
def test_sa_backward_accepts_prototype_chunks(kw):
    # supported shapes pass the host checks and stop only at the missing device
    assert bwd(sa_desc(**kw)) == L.SKA_ERR_CUDA


def test_sa_backward_pointer_checks():
    d = sa_desc()
    assert bwd(d, dq=None) == INVALID
    assert bwd(d, dsk=None) == INVALID
    assert bwd(d, lse=None) == INVALID
    assert bwd(d, dk=None) == INVALID
    assert bwd(sa_desc(norm=L.SKA_NORM_TOKEN), sk=None) == INVALID  # D_j needs the sketch
    assert bwd(d, dv=10 * A + 4) == INVALID


@pytest.mark.parametrize("kw,code", [
    ({"num_heads": 0}, INVALID), ({"num_sketch": -1}, INVALID), ({"total_hist": -1}, INVALID),
    ({"scale": 0.0}, INVALID), ({"head_dim": 32}, UNSUP),
    ({"num_heads": 1 << 16, "total_hist": (1 << 31) - 1}, INVALID),
])
def test_stca_rejects_bad_descriptors(kw, code):
    assert stca(stca_desc(**kw)) == code


def test_stca_pointer_checks():
    d = stca_desc()
    assert stca(None) == INVALID
    assert stca(d, q=None) == INVALID
    assert stca(d, kh=None) == INVALID
    assert stca(d, ks=None) == INVALID
    assert stca(stca_desc(num_sketch=0), ks=None, vs=None) != INVALID  # no sketch rows: no sketch pointers needed
    assert stca(d, out=8 * A + 4) == INVALID
    assert stca(d, kvl=2 * A + 2) == INVALID


def test_valid_call_without_a_device_reports_cuda_error():
    """Arguments that pass every host check reach the device query, which fails loudly here."""
    import torch
    if torch.cuda.is_available():
        pytest.skip("a device is present")
    assert fwd(sa_desc()) == L.SKA_ERR_CUDA
    assert b"cudaGetDevice" in L.lib().ska_last_error_string()
    assert fwd(sa_desc(), mass=11 * A) == L.SKA_ERR_CUDA  # the mass output passes the host checks
    assert L.lib().sa_forward_noalloc_read_status(None) == L.SKA_ERR_CUDA
    assert bwd(sa_desc()) == L.SKA_ERR_CUDA
    assert stca(stca_desc()) == L.SKA_ERR_CUDA
    assert L.lib().sa_forward_workspace_size(ctypes.byref(sa_desc())) == 0


def test_debug_and_timing_hooks_are_host_only():
    lib = L.lib()
    lib.ska_set_debug(1_000_000, 0)
    lib.ska_set_debug(0, 0)  # back to the default budget
    lib.ska_set_timing_events(None, None)


def refine_desc(**kw):
    f = dict(num_users=2, num_heads=2, num_protos=300, head_dim=128, ffn_dim=256, eps=1e-5, x_tilde_shared=0,
             reserved=0)
    f.update(kw)
    return L.RefineDesc(**f)


REFINE_ARGS = ["xt", "xh", "w1", "wg", "w2", "g1", "b1", "g2", "b2", "wq", "out", "bar", "bf", "q", "ws"]


def refine(d, **kw):
    ptrs = {n: (i + 20) * A for i, n in enumerate(REFINE_ARGS)}
    ws_bytes = kw.pop("ws_bytes", 256)
    ptrs.update(kw)
    return L.lib().sa_refine(ctypes.byref(d) if d is not None else None, *[ptrs[n] for n in REFINE_ARGS],
                             ws_bytes, None)


@pytest.mark.parametrize("kw,code", [
    ({"num_heads": 0}, INVALID), ({"num_protos": 0}, INVALID), ({"num_users": -1}, INVALID),
    ({"eps": 0.0}, INVALID), ({"eps": float("inf")}, INVALID), ({"eps": float("nan")}, INVALID),
    ({"head_dim": 96, "ffn_dim": 192}, UNSUP), ({"ffn_dim": 128}, UNSUP), ({"head_dim": 64, "ffn_dim": 256}, UNSUP),
    ({"num_users": 1 << 12, "num_heads": 64, "num_protos": 64}, INVALID),  # B H k d >= 2^31
])
def test_refine_rejects_bad_descriptors(kw, code):
    d = refine_desc(**kw)
    assert refine(d) == code
    assert L.lib().sa_refine_workspace_size(ctypes.byref(d)) == 0


def test_refine_pointer_checks():
    d = refine_desc()
    assert L.lib().sa_refine_workspace_size(ctypes.byref(d)) == 256
    assert refine(None) == INVALID
    for n in ("xt", "xh", "w1", "wg", "w2", "out", "ws"):
        assert refine(d, **{n: None}) == INVALID, n
    assert refine(d, wq=None) == INVALID                 # W_Q and q_next come together
    assert refine(d, q=None) == INVALID
    assert refine(d, g1=40 * A + 4) == INVALID           # 16-byte alignment
    assert refine(d, ws=41 * A + 16) == INVALID          # 256-byte workspace alignment
    assert refine(d, ws_bytes=255) == L.SKA_ERR_WORKSPACE_TOO_SMALL
    assert refine(d, out=20 * A + 64) == INVALID         # the output overlaps x_tilde
    assert refine(d, bar=30 * A + 1024) == INVALID       # x_bar overlaps x_next
    assert refine(d, q=31 * A + 512) == INVALID          # q_next overlaps x_bar
    assert refine(d, ws=22 * A) == INVALID               # the workspace overlaps W_1
    # B = 0: nothing to do, no pointer is looked at
    assert refine(refine_desc(num_users=0), xt=None, xh=None, out=None, ws=None) == L.SKA_OK


def project(B=2, H=2, k=300, d=128, **kw):
    names = ["x", "wq", "q", "ws"]
    ptrs = {n: (i + 50) * A for i, n in enumerate(names)}
    ws_bytes = kw.pop("ws_bytes", 256)
    ptrs.update(kw)
    return L.lib().sa_project_queries(B, H, k, d, *[ptrs[n] for n in names], ws_bytes, None)


def test_project_queries_host_checks():
    assert project(H=0) == INVALID
    assert project(k=0) == INVALID
    assert project(B=-1) == INVALID
    assert project(d=96) == UNSUP
    assert project(B=1 << 12, H=64, k=64) == INVALID
    assert project(B=0, x=None, wq=None, q=None, ws=None) == L.SKA_OK
    for n in ("x", "wq", "q", "ws"):
        assert project(**{n: None}) == INVALID, n
    assert project(q=50 * A + 16) == INVALID             # q overlaps x
    assert project(x=50 * A + 8) == INVALID              # alignment
    assert project(ws_bytes=100) == L.SKA_ERR_WORKSPACE_TOO_SMALL


def test_refine_without_a_device_reports_cuda_error():
    import torch
    if torch.cuda.is_available():
        pytest.skip("a device is present")
    d = refine_desc()
    # optional outputs, W_Q and LayerNorm vectors may be NULL
    assert refine(d, g1=None, b1=None, g2=None, b2=None, bar=None, bf=None, wq=None, q=None) == L.SKA_ERR_CUDA
    assert refine(refine_desc(head_dim=64, ffn_dim=128)) == L.SKA_ERR_CUDA
    assert refine(refine_desc(x_tilde_shared=1)) == L.SKA_ERR_CUDA
    assert project() == L.SKA_ERR_CUDA


STCA_BWD_ARGS = ["q", "cut", "kh", "vh", "cuh", "kvl", "ks", "vs", "out", "lse", "do", "dq", "dkh", "dvh", "dks",
                 "dvs", "ws"]


def stca_bwd(desc, **kw):
    ptrs = {n: (i + 70) * A for i, n in enumerate(STCA_BWD_ARGS)}
    ptrs["kvl"] = None
    ws_bytes = kw.pop("ws_bytes", 1 << 30)
    ptrs.update(kw)
    return L.lib().stca_backward(ctypes.byref(desc) if desc is not None else None,
                                 *[ptrs[n] for n in STCA_BWD_ARGS], ws_bytes, None)


def test_stca_backward_host_checks():
    d = stca_desc()
    need = L.lib().stca_backward_workspace_size(ctypes.byref(d))
    assert need >= 256 + 100 * 2 * 4  # header, prefixes, one delta per (target, head)
    assert stca_bwd(None) == INVALID
    assert stca_bwd(stca_desc(head_dim=32)) == UNSUP
    assert stca_bwd(stca_desc(num_heads=0)) == INVALID
    for n in ("q", "out", "lse", "do", "dq", "kh", "dkh", "dvs", "ws"):
        assert stca_bwd(d, **{n: None}) == INVALID, n
    assert stca_bwd(stca_desc(num_sketch=0), ks=None, vs=None, dks=None, dvs=None) != INVALID
    assert stca_bwd(d, ws_bytes=need - 1) == L.SKA_ERR_WORKSPACE_TOO_SMALL
    assert stca_bwd(d, dq=70 * A + 64) == INVALID      # dq overlaps q
    assert stca_bwd(d, dvh=82 * A + 256) == INVALID    # dv_hist overlaps dk_hist
    assert stca_bwd(d, kvl=2 * A + 2) == INVALID       # int32 alignment
    assert stca_bwd(stca_desc(num_users=0, total_targets=0, total_hist=0), q=None, cut=None, ws=None) == L.SKA_OK


def test_stca_backward_without_a_device_reports_cuda_error():
    import torch
    if torch.cuda.is_available():
        pytest.skip("a device is present")
    assert stca_bwd(stca_desc()) == L.SKA_ERR_CUDA


def diag(desc, mw=12 * A, renorm=0, mass=11 * A, **kw):
    args = dict(q=A, k=2 * A, v=3 * A, cu=4 * A, su=None, sk=5 * A, lse=6 * A, ws=256 * A)
    args.update(kw)
    return L.lib().sa_forward_diag(ctypes.byref(desc), args["q"], args["k"], args["v"], args["cu"], args["su"],
                                   args["sk"], args["lse"], mass, mw, renorm, args["ws"], 1 << 30, None)


def test_forward_diag_and_histogram_host_checks():
    assert diag(sa_desc(norm=L.SKA_NORM_TOKEN)) == UNSUP          # prototype-wise only
    assert diag(sa_desc(norm=L.SKA_NORM_TOKEN), mw=None, renorm=1) == UNSUP
    assert diag(sa_desc(), renorm=1, mass=None) == INVALID        # the divisors are the mass output
    assert diag(sa_desc(), mw=12 * A + 8) == INVALID              # alignment
    assert diag(sa_desc(), mw=5 * A + 64) == INVALID              # overlaps the sketch
    h = L.lib().sa_weight_histogram
    assert h(None, 10, 4, 20 * A, None) == INVALID
    assert h(21 * A, 10, 0, 20 * A, None) == INVALID
    assert h(21 * A, 10, 5000, 20 * A, None) == INVALID
    assert h(21 * A, -1, 4, 20 * A, None) == INVALID
    assert h(21 * A, 10, 4, 21 * A + 8, None) == INVALID          # counts overlap the values
    import torch
    if not torch.cuda.is_available():
        assert diag(sa_desc()) == L.SKA_ERR_CUDA
        assert h(21 * A, 10, 4, 20 * A, None) == L.SKA_ERR_CUDA


def test_cache_host_checks():
    lib = L.lib()
    good = L.CacheDesc(64, 8, 16, 0, 100)
    nb = lib.sa_cache_bytes(ctypes.byref(good))
    assert nb >= 256 + 64 * 8 * (32 + 16 * 4)
    for bad in (L.CacheDesc(48, 8, 16, 0, 100), L.CacheDesc(64, 33, 16, 0, 100), L.CacheDesc(64, 8, 6, 0, 100),
                L.CacheDesc(64, 8, 16, 0, -1), L.CacheDesc(0, 8, 16, 0, 1)):
        assert lib.sa_cache_bytes(ctypes.byref(bad)) == 0
        assert lib.sa_cache_init(ctypes.byref(bad), 90 * A, nb, None) == INVALID
    assert lib.sa_cache_init(ctypes.byref(good), 90 * A, nb - 1, None) == L.SKA_ERR_WORKSPACE_TOO_SMALL
    assert lib.sa_cache_init(ctypes.byref(good), 90 * A + 128, nb, None) == INVALID
    put = lambda **kw: lib.sa_cache_put(ctypes.byref(good), kw.get("c", 90 * A), nb, kw.get("k", 91 * A),  # noqa: E731
                                        kw.get("r", 92 * A), kw.get("n", 10), 5, kw.get("s", 93 * A), None)
    assert put(n=-1) == INVALID
    assert put(n=0, k=None, r=None, s=None) == L.SKA_OK
    assert put(k=91 * A + 4) == INVALID                 # keys are 8-byte aligned
    assert put(r=92 * A + 8) == INVALID                 # rows 16-byte aligned
    assert put(s=92 * A + 64) == INVALID                # slots overlap the rows
    get = lambda **kw: lib.sa_cache_get(ctypes.byref(good), 90 * A, nb, kw.get("k", 91 * A), 10, 5,  # noqa: E731
                                        kw.get("o", 92 * A), kw.get("h", 93 * A), None)
    assert get(o=90 * A + 1024) == INVALID              # output overlaps the cache
    assert get(h=None) == INVALID
    import torch
    if not torch.cuda.is_available():
        assert put() == L.SKA_ERR_CUDA and get() == L.SKA_ERR_CUDA
