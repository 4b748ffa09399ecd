"""The torch binding's argument checks, without a GPU. The C ABI takes every size from its
descriptor and cannot see a buffer that does not match it, so the binding compares the tensors with
one another before it passes any pointer on; each mismatch below must raise ValueError on the host
(CPU tensors are enough: the shape and dtype checks come before the device checks)."""
import pytest
import torch

from sketch_attention_flashsa_b200 import api

B, T, H, D, K = 3, 50, 2, 64, 32
bf, f32, i32 = torch.bfloat16, torch.float32, torch.int32


def sa_args(**over):
    a = dict(q=torch.zeros(H, K, D, dtype=bf), k=torch.zeros(T, H, D, dtype=bf), v=torch.zeros(T, H, D, dtype=bf),
             cu_seqlens=torch.tensor([0, 10, 30, 50], dtype=i32), seqused=None)
    a.update(over)
    return a


def fwd(norm="proto", **over):
    a = sa_args(**{k: v for k, v in over.items() if k in ("q", "k", "v", "cu_seqlens", "seqused")})
    kw = {k: v for k, v in over.items() if k not in a}
    return api.sa_forward(a["q"], a["k"], a["v"], a["cu_seqlens"], a["seqused"], norm=norm, **kw)


@pytest.mark.parametrize("over,msg", [
    (dict(q=torch.zeros(H, K, D, dtype=f32)), "share one dtype"),            # fp32 q with bf16 k, v
    (dict(v=torch.zeros(T, H, D, dtype=f32)), "share one dtype"),
    (dict(k=torch.zeros(T, H, D, dtype=torch.float16)), "dtype"),           # unsupported dtype
    (dict(v=torch.zeros(T + 1, H, D, dtype=bf)), "shape"),                  # v rows differ from k
    (dict(q=torch.zeros(H + 1, K, D, dtype=bf)), "heads"),                  # q heads differ from k
    (dict(q=torch.zeros(H, K, 128, dtype=bf)), "head_dim"),                 # q head_dim differs
    (dict(q=torch.zeros(B + 1, H, K, D, dtype=bf)), "users"),               # per-user q, wrong user count
    (dict(k=torch.zeros(T, H * D, dtype=bf), v=torch.zeros(T, H * D, dtype=bf)), "k must be"),
    (dict(cu_seqlens=torch.tensor([0, 10, 50], dtype=torch.int64)), "cu_seqlens"),
    (dict(seqused=torch.tensor([1, 2], dtype=i32)), "seqused"),             # B entries needed
    (dict(out=torch.zeros(B, H, K, D + 1, dtype=f32)), "out"),             # sketch output shape
    (dict(out=torch.zeros(B, H, K, D, dtype=bf)), "dtype"),                 # sketch output dtype
    (dict(lse_out=torch.zeros(B, H, K, dtype=f32)), "lse_out"),            # proto lse is [T, H]
    (dict(mass_out=torch.zeros(B, H, K + 1, dtype=f32)), "mass_out"),
])
def test_sa_forward_rejects_mismatched_tensors(over, msg):
    with pytest.raises(ValueError, match=msg):
        fwd(**over)


def test_token_lse_shape_is_per_prototype():
    with pytest.raises(ValueError, match="lse_out"):
        fwd(norm="token", lse_out=torch.zeros(T, H, dtype=f32))


def test_noalloc_needs_preallocated_outputs():
    a = sa_args()
    with pytest.raises(ValueError, match="preallocated"):
        api.sa_forward_noalloc(a["q"], a["k"], a["v"], a["cu_seqlens"])
    with pytest.raises(ValueError, match="out"):
        api.sa_forward_noalloc(a["q"], a["k"], a["v"], a["cu_seqlens"], out=torch.zeros(B, H, K, 3, dtype=f32))


def bwd(norm="proto", **over):
    a = sa_args(**{k: v for k, v in over.items() if k in ("q", "k", "v", "cu_seqlens", "seqused")})
    lse = over.get("lse", torch.zeros((T, H) if norm == "proto" else (B, H, K), dtype=f32))
    ds = over.get("dsketch", torch.zeros(B, H, K, D, dtype=bf))
    sk = over.get("sketch", None)
    return api.sa_backward(a["q"], a["k"], a["v"], a["cu_seqlens"], a["seqused"], lse, ds, sk, norm=norm)


@pytest.mark.parametrize("over,msg", [
    (dict(q=torch.zeros(H, K, D, dtype=f32), k=torch.zeros(T, H, D, dtype=f32),
          v=torch.zeros(T, H, D, dtype=f32)), "dtype"),                     # the backward is bf16 only
    (dict(dsketch=torch.zeros(B, H, K, D, dtype=f32)), "dsketch"),
    (dict(dsketch=torch.zeros(B, H, K + 16, D, dtype=bf)), "dsketch"),
    (dict(lse=torch.zeros(T + 1, H, dtype=f32)), "lse"),
    (dict(sketch=torch.zeros(B, H, K, D, dtype=bf)), "sketch"),
    (dict(v=torch.zeros(T, H + 1, D, dtype=bf)), "shape"),
])
def test_sa_backward_rejects_mismatched_tensors(over, msg):
    with pytest.raises(ValueError, match=msg):
        bwd(**over)


def test_token_backward_needs_the_sketch():
    with pytest.raises(ValueError, match="sketch"):
        bwd(norm="token")


Tq, Th, KS = 40, 70, 16


def stca(**over):
    a = dict(q=torch.zeros(Tq, H, D, dtype=bf), cu_targets=torch.tensor([0, 15, 40], dtype=i32),
             k_hist=torch.zeros(Th, H, D, dtype=bf), v_hist=torch.zeros(Th, H, D, dtype=bf),
             cu_hist=torch.tensor([0, 30, 70], dtype=i32), k_sk=torch.zeros(2, H, KS, D, dtype=bf),
             v_sk=torch.zeros(2, H, KS, D, dtype=bf))
    kw = {k: v for k, v in over.items() if k not in a}
    a.update({k: v for k, v in over.items() if k in a})
    return api.stca_forward(a["q"], a["cu_targets"], a["k_hist"], a["v_hist"], a["cu_hist"], a["k_sk"], a["v_sk"],
                            scale=0.125, max_targets=25, **kw)


@pytest.mark.parametrize("over,msg", [
    (dict(q=torch.zeros(Tq, H, D, dtype=f32)), "dtype"),
    (dict(k_hist=torch.zeros(Th, H + 1, D, dtype=bf)), "k_hist"),
    (dict(v_hist=torch.zeros(Th + 3, H, D, dtype=bf)), "v_hist"),
    (dict(k_sk=torch.zeros(3, H, KS, D, dtype=bf)), "k_sk"),                # one sketch block per user
    (dict(v_sk=torch.zeros(2, H, KS + 1, D, dtype=bf)), "v_sk"),
    (dict(v_sk=None), "together"),
    (dict(cu_hist=torch.tensor([0, 70], dtype=i32)), "cu_hist"),
    (dict(target_kv_len=torch.zeros(Tq + 1, dtype=i32)), "target_kv_len"),
    (dict(out=torch.zeros(Tq, H, D + 1, dtype=f32)), "out"),
    (dict(lse_out=torch.zeros(Tq, H + 1, dtype=f32)), "lse_out"),
])
def test_stca_rejects_mismatched_tensors(over, msg):
    with pytest.raises(ValueError, match=msg):
        stca(**over)


def stca_bwd(**over):
    a = dict(q=torch.zeros(Tq, H, D, dtype=bf), cu_targets=torch.tensor([0, 15, 40], dtype=i32),
             k_hist=torch.zeros(Th, H, D, dtype=bf), v_hist=torch.zeros(Th, H, D, dtype=bf),
             cu_hist=torch.tensor([0, 30, 70], dtype=i32), k_sk=torch.zeros(2, H, KS, D, dtype=bf),
             v_sk=torch.zeros(2, H, KS, D, dtype=bf), out=torch.zeros(Tq, H, D, dtype=f32),
             lse=torch.zeros(Tq, H, dtype=f32), dout=torch.zeros(Tq, H, D, dtype=bf))
    kw = {k: v for k, v in over.items() if k not in a}
    a.update({k: v for k, v in over.items() if k in a})
    return api.stca_backward(a["q"], a["cu_targets"], a["k_hist"], a["v_hist"], a["cu_hist"], a["k_sk"], a["v_sk"],
                             a["out"], a["lse"], a["dout"], scale=0.125, **kw)


@pytest.mark.parametrize("over,msg", [
    (dict(q=torch.zeros(Tq, H, D, dtype=f32)), "dtype"),
    (dict(dout=torch.zeros(Tq, H, D, dtype=f32)), "dtype"),
    (dict(q=torch.zeros(Tq, H * D, dtype=bf)), "q must be"),
    (dict(cu_targets=torch.tensor([0, 15, 40], dtype=torch.int64)), "cu_targets"),
    (dict(cu_hist=torch.tensor([0, 70], dtype=i32)), "cu_hist"),
    (dict(k_hist=torch.zeros(Th, H + 1, D, dtype=bf)), "k_hist"),
    (dict(v_hist=torch.zeros(Th + 1, H, D, dtype=bf)), "v_hist"),
    (dict(v_sk=None), "together"),
    (dict(k_sk=torch.zeros(3, H, KS, D, dtype=bf)), "k_sk"),
    (dict(out=torch.zeros(Tq, H, D + 1, dtype=f32)), "out"),
    (dict(lse=torch.zeros(Tq + 1, H, dtype=f32)), "lse"),
    (dict(dout=torch.zeros(Tq, H, D + 1, dtype=bf)), "dout"),
    (dict(target_kv_len=torch.zeros(Tq, dtype=torch.int64)), "target_kv_len"),
])
def test_stca_backward_rejects_mismatched_tensors(over, msg):
    with pytest.raises(ValueError, match=msg):
        stca_bwd(**over)


KR, F = 128, 2 * D


def refine(**over):
    a = dict(x_tilde=torch.zeros(B, H, KR, D, dtype=f32), x_hat=torch.zeros(B, H, KR, D, dtype=f32),
             w1=torch.zeros(H, D, F, dtype=bf), wg=torch.zeros(H, D, F, dtype=bf), w2=torch.zeros(H, F, D, dtype=bf))
    kw = {k: v for k, v in over.items() if k not in a}
    a.update({k: v for k, v in over.items() if k in a})
    return api.sa_refine(a["x_tilde"], a["x_hat"], a["w1"], a["wg"], a["w2"], **kw)


@pytest.mark.parametrize("over,msg", [
    (dict(x_hat=torch.zeros(H, KR, D, dtype=f32)), "x_hat must be"),
    (dict(x_tilde=torch.zeros(B, H, KR + 1, D, dtype=f32)), "x_tilde"),
    (dict(x_tilde=torch.zeros(H + 1, KR, D, dtype=f32)), "x_tilde"),       # shared rows: [H, k, d]
    (dict(w1=torch.zeros(H, D + 1, F, dtype=bf)), "w1 must be"),
    (dict(wg=torch.zeros(H, D, F + 8, dtype=bf)), "wg"),
    (dict(w2=torch.zeros(H, D, F, dtype=bf)), "w2"),                         # [H, F, d], not [H, d, F]
    (dict(w_q_next=torch.zeros(H, D, D + 1, dtype=bf)), "w_q_next"),
    (dict(gamma1=torch.zeros(H, D + 1, dtype=f32)), "gamma1"),
    (dict(beta2=torch.zeros(H + 1, D, dtype=f32)), "beta2"),
    (dict(out=torch.zeros(B, H, KR, D + 1, dtype=f32)), "out"),
    (dict(x_hat=torch.zeros(B, H, KR, D, dtype=bf), x_tilde=torch.zeros(B, H, KR, D, dtype=bf)), "dtype"),
    (dict(w1=torch.zeros(H, D, F, dtype=f32)), "dtype"),
])
def test_refine_rejects_mismatched_tensors(over, msg):
    with pytest.raises(ValueError, match=msg):
        refine(**over)


@pytest.mark.parametrize("x,w_q,out,msg", [
    (torch.zeros(KR, D, dtype=f32), torch.zeros(H, D, D, dtype=bf), None, "x must be"),
    (torch.zeros(H, KR, D, dtype=f32), torch.zeros(H + 1, D, D, dtype=bf), None, "w_q"),
    (torch.zeros(B, H, KR, D, dtype=f32), torch.zeros(H, D, D, dtype=bf), torch.zeros(B, H, KR, D + 1, dtype=bf),
     "out"),
    (torch.zeros(H, KR, D, dtype=bf), torch.zeros(H, D, D, dtype=bf), None, "dtype"),
    (torch.zeros(H, KR, D, dtype=f32), torch.zeros(H, D, D, dtype=f32), None, "dtype"),
])
def test_project_queries_rejects_mismatched_tensors(x, w_q, out, msg):
    with pytest.raises(ValueError, match=msg):
        api.project_queries(x, w_q, out=out)


def test_cache_keys_have_the_c_layout():
    """cache_keys packs the fields into the 24 bytes of ska_cache_key (user id, version and
    configuration as two 32-bit words, timestamp), with scalars broadcast over the batch."""
    import ctypes
    from sketch_attention_flashsa_b200 import _lib
    keys = api.cache_keys([5, 2**40 + 3], 0xFFFFFFFE, [0x12345678, 0x9ABCDEF0], -7, device="cpu")
    assert keys.dtype == torch.int64 and tuple(keys.shape) == (2, 3)
    want = b"".join(bytes(_lib.CacheKey(u, 0xFFFFFFFE, c, -7))
                    for u, c in ((5, 0x12345678), (2**40 + 3, 0x9ABCDEF0)))
    assert ctypes.sizeof(_lib.CacheKey) == 24
    assert keys.numpy().tobytes() == want


@pytest.mark.parametrize("call,msg", [
    (lambda: api.weight_histogram(torch.zeros(10, dtype=torch.float64), 8), "dtype"),
    (lambda: api.sa_forward_diag(torch.zeros(H, K, D, dtype=f32), torch.zeros(T, H, D, dtype=bf),
                                 torch.zeros(T, H, D, dtype=bf), torch.tensor([0, 10, 30, 50], dtype=i32)),
     "share one dtype"),
    (lambda: api.sa_forward_diag(torch.zeros(H + 1, K, D, dtype=bf), torch.zeros(T, H, D, dtype=bf),
                                 torch.zeros(T, H, D, dtype=bf), torch.tensor([0, 10, 30, 50], dtype=i32)), "heads"),
])
def test_diagnostics_reject_mismatched_tensors(call, msg):
    with pytest.raises(ValueError, match=msg):
        call()
