"""Torch-facing binding of the C ABI: takes device tensors, passes their pointers and the
current CUDA stream to libska.so, and returns the outputs. No computation happens here."""
from __future__ import annotations

import ctypes
from typing import Optional

import torch

from . import _lib
from ._lib import RefineDesc, SaDesc, SkaError, StcaDesc

_NORMS = {"proto": _lib.SKA_NORM_PROTO, "token": _lib.SKA_NORM_TOKEN,
          _lib.SKA_NORM_PROTO: _lib.SKA_NORM_PROTO, _lib.SKA_NORM_TOKEN: _lib.SKA_NORM_TOKEN}


def _ptr(t: Optional[torch.Tensor]):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else ctypes.c_void_p(0)


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _dev_tensor(name, t, dtypes):
    if t is None:
        return
    if t.dtype not in dtypes:
        raise ValueError(f"{name} has dtype {t.dtype}, expected one of {dtypes}")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _dtypes(pairs, dtypes):
    """Dtype checks of several tensors, ahead of any device check (a wrong dtype is reported as such
    wherever the tensor lives)."""
    for name, t in pairs:
        if t is not None and t.dtype not in dtypes:
            raise ValueError(f"{name} has dtype {t.dtype}, expected one of {dtypes}")


def _shape(name, t, want):
    if t is not None and tuple(t.shape) != tuple(want):
        raise ValueError(f"{name}: shape {tuple(t.shape)}, expected {tuple(want)}")


def _check_sa_inputs(q, k, v, cu_seqlens, seqused, dtypes):
    """Shapes and dtypes of an SA call's inputs, checked against one another on the host (the C ABI
    takes the sizes from the descriptor and cannot see a mismatched buffer)."""
    for name, t in (("q", q), ("k", k), ("v", v)):
        if t.dtype not in dtypes:
            raise ValueError(f"{name} has dtype {t.dtype}, expected one of {dtypes}")
    if not (q.dtype == k.dtype == v.dtype):
        raise ValueError(f"q, k and v must share one dtype (got {q.dtype}, {k.dtype}, {v.dtype})")
    if k.dim() != 3:
        raise ValueError(f"k must be [T, H, d], got shape {tuple(k.shape)}")
    _shape("v", v, k.shape)
    if q.dim() not in (3, 4):
        raise ValueError(f"q must be [H, k, d] or [B, H, k, d], got shape {tuple(q.shape)}")
    if cu_seqlens.dim() != 1 or cu_seqlens.numel() < 1 or cu_seqlens.dtype != torch.int32:
        raise ValueError("cu_seqlens must be a 1-D int32 tensor of B + 1 offsets")
    B = cu_seqlens.numel() - 1
    H, d = k.shape[1], k.shape[2]
    if q.shape[-3] != H or q.shape[-1] != d:
        raise ValueError(f"q {tuple(q.shape)} does not match k's heads {H} and head_dim {d}")
    if q.dim() == 4 and q.shape[0] != B:
        raise ValueError(f"per-user q has {q.shape[0]} users, cu_seqlens describes {B}")
    if seqused is not None:
        if seqused.dtype != torch.int32 or tuple(seqused.shape) != (B,):
            raise ValueError(f"seqused must be int32 of shape ({B},)")
    return B, H, q.shape[-2], d


def _check(rc: int, what: str):
    if rc != _lib.SKA_OK:
        raise SkaError(rc, what)


def sa_desc(q, k, cu_seqlens, *, scale, norm, max_seqlen=0) -> SaDesc:
    per_user = q.dim() == 4
    d = SaDesc()
    d.num_users = cu_seqlens.numel() - 1
    d.num_heads = k.shape[1]
    d.head_dim = k.shape[2]
    d.num_protos = q.shape[-2]
    d.total_tokens = k.shape[0]
    d.max_seqlen = int(max_seqlen)
    d.scale = float(scale)
    d.norm = _NORMS[norm]
    d.in_dtype = _lib.SKA_F32 if q.dtype == torch.float32 else _lib.SKA_BF16
    d.q_per_user = 1 if per_user else 0
    d.reserved = 0
    return d


def sa_forward_workspace_size(desc: SaDesc) -> int:
    return int(_lib.lib().sa_forward_workspace_size(ctypes.byref(desc)))


def sa_forward(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, cu_seqlens: torch.Tensor,
               seqused: Optional[torch.Tensor] = None, *, scale: float = 1.0, norm="proto",
               want_lse: bool = True, want_mass: bool = False, workspace: Optional[torch.Tensor] = None,
               out: Optional[torch.Tensor] = None, lse_out: Optional[torch.Tensor] = None,
               mass_out: Optional[torch.Tensor] = None, stream=None):
    """Sketch Attention forward (SequenceO1 §3.1 Eq. (7)-(9), FlashSA §4.4).

    q [H,k,d] or [B,H,k,d]; k, v [T,H,d] (bf16, or fp32 rounded to bf16 on the device; all three
    of one dtype); cu_seqlens int32 [B+1]; seqused int32 [B] or None. out / lse_out / mass_out:
    optional preallocated outputs. Returns (sketch fp32 [B,H,k,d], lse or None, mass or None):
    lse is [T,H] (prototype-wise) or [B,H,k] (token-wise); mass [B,H,k] = sum_i A[j,i].
    """
    B, H, kp, D = _check_sa_inputs(q, k, v, cu_seqlens, seqused, (torch.bfloat16, torch.float32))
    nid = _NORMS[norm]
    T = k.shape[0]
    _shape("out", out, (B, H, kp, D))
    _shape("lse_out", lse_out, (T, H) if nid == _lib.SKA_NORM_PROTO else (B, H, kp))
    _shape("mass_out", mass_out, (B, H, kp))
    for name, t in (("out", out), ("lse_out", lse_out), ("mass_out", mass_out)):
        _dev_tensor(name, t, (torch.float32,))
    for name, t in (("q", q), ("k", k), ("v", v)):
        _dev_tensor(name, t, (torch.bfloat16, torch.float32))
    _dev_tensor("cu_seqlens", cu_seqlens, (torch.int32,))
    _dev_tensor("seqused", seqused, (torch.int32,))
    desc = sa_desc(q, k, cu_seqlens, scale=scale, norm=norm)
    dev = k.device
    need = sa_forward_workspace_size(desc)
    if need == 0 and B > 0:
        raise SkaError(_lib.SKA_ERR_UNSUPPORTED, "sa_forward_workspace_size")
    if workspace is None or workspace.numel() < need:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=dev)
    sketch = out if out is not None else torch.empty((B, H, kp, D), dtype=torch.float32, device=dev)
    lse = None
    if want_lse or lse_out is not None:
        shape = (T, H) if desc.norm == _lib.SKA_NORM_PROTO else (B, H, kp)
        lse = lse_out if lse_out is not None else torch.empty(shape, dtype=torch.float32, device=dev)
    mass = None
    if want_mass or mass_out is not None:
        mass = mass_out if mass_out is not None else torch.empty((B, H, kp), dtype=torch.float32, device=dev)
    rc = _lib.lib().sa_forward(ctypes.byref(desc), _ptr(q), _ptr(k), _ptr(v), _ptr(cu_seqlens),
                               _ptr(seqused), _ptr(sketch), _ptr(lse), _ptr(mass), _ptr(workspace),
                               ctypes.c_size_t(workspace.numel()), _stream(stream))
    _check(rc, "sa_forward")
    return sketch, lse, mass


def sa_forward_diag(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, cu_seqlens: torch.Tensor,
                    seqused: Optional[torch.Tensor] = None, *, scale: float = 1.0, want_max_weight: bool = True,
                    renormalize: bool = False, workspace: Optional[torch.Tensor] = None, stream=None):
    """Prototype-wise SA forward with the allocation diagnostics: each token's largest weight
    max_j A[j,i] (SequenceO1 §5.1 Fig. 3; -1 on padding rows) and, with `renormalize`, the sketch
    rows divided by their mass (the Slot-Attention weighted mean, §2.4).
    Returns (sketch [B,H,k,d], lse [T,H], mass [B,H,k], max_weight [T,H] or None)."""
    B, H, kp, D = _check_sa_inputs(q, k, v, cu_seqlens, seqused, (torch.bfloat16, torch.float32))
    T = k.shape[0]
    for name, t in (("q", q), ("k", k), ("v", v)):
        _dev_tensor(name, t, (torch.bfloat16, torch.float32))
    _dev_tensor("cu_seqlens", cu_seqlens, (torch.int32,))
    _dev_tensor("seqused", seqused, (torch.int32,))
    desc = sa_desc(q, k, cu_seqlens, scale=scale, norm="proto")
    dev = k.device
    need = sa_forward_workspace_size(desc)
    if need == 0 and B > 0:
        raise SkaError(_lib.SKA_ERR_UNSUPPORTED, "sa_forward_workspace_size")
    if workspace is None or workspace.numel() < need:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=dev)
    sketch = torch.empty((B, H, kp, D), dtype=torch.float32, device=dev)
    lse = torch.empty((T, H), dtype=torch.float32, device=dev)
    mass = torch.empty((B, H, kp), dtype=torch.float32, device=dev)
    mw = torch.empty((T, H), dtype=torch.float32, device=dev) if want_max_weight else None
    rc = _lib.lib().sa_forward_diag(ctypes.byref(desc), _ptr(q), _ptr(k), _ptr(v), _ptr(cu_seqlens), _ptr(seqused),
                                    _ptr(sketch), _ptr(lse), _ptr(mass), _ptr(mw), 1 if renormalize else 0,
                                    _ptr(workspace), ctypes.c_size_t(workspace.numel()), _stream(stream))
    _check(rc, "sa_forward_diag")
    return sketch, lse, mass, mw


def weight_histogram(values: torch.Tensor, bins: int, *, out: Optional[torch.Tensor] = None, stream=None):
    """Counts of the values in `bins` equal bins over [0, 1] (1.0 in the last; negative values and
    NaN skipped), as int32 on the device."""
    _dev_tensor("values", values, (torch.float32,))
    counts = torch.empty(bins, dtype=torch.int32, device=values.device) if out is None else out
    _shape("out", counts, (bins,))
    _dev_tensor("out", counts, (torch.int32,))
    rc = _lib.lib().sa_weight_histogram(_ptr(values), int(values.numel()), int(bins), _ptr(counts), _stream(stream))
    _check(rc, "sa_weight_histogram")
    return counts


def sa_forward_noalloc(q, k, v, cu_seqlens, seqused=None, *, scale: float = 1.0, norm="proto", out=None,
                       lse_out=None, mass_out=None, stream=None):
    """sa_forward for callers that cannot allocate device memory: scratch comes from a fixed array
    inside libska.so (sa_forward_noalloc_scratch_bytes()). The outputs must be preallocated."""
    B, H, kp, D = _check_sa_inputs(q, k, v, cu_seqlens, seqused, (torch.bfloat16, torch.float32))
    nid = _NORMS[norm]
    if out is None:
        raise ValueError("sa_forward_noalloc writes into a preallocated out")
    _shape("out", out, (B, H, kp, D))
    _shape("lse_out", lse_out, (k.shape[0], H) if nid == _lib.SKA_NORM_PROTO else (B, H, kp))
    _shape("mass_out", mass_out, (B, H, kp))
    for name, t in (("out", out), ("lse_out", lse_out), ("mass_out", mass_out)):
        _dev_tensor(name, t, (torch.float32,))
    for name, t in (("q", q), ("k", k), ("v", v)):
        _dev_tensor(name, t, (torch.bfloat16, torch.float32))
    _dev_tensor("cu_seqlens", cu_seqlens, (torch.int32,))
    _dev_tensor("seqused", seqused, (torch.int32,))
    desc = sa_desc(q, k, cu_seqlens, scale=scale, norm=norm)
    rc = _lib.lib().sa_forward_noalloc(ctypes.byref(desc), _ptr(q), _ptr(k), _ptr(v), _ptr(cu_seqlens),
                                       _ptr(seqused), _ptr(out), _ptr(lse_out), _ptr(mass_out), _stream(stream))
    _check(rc, "sa_forward_noalloc")
    return out, lse_out, mass_out


def read_noalloc_status(stream=None) -> int:
    """Device status of the last sa_forward_noalloc call on this device (synchronises, then clears)."""
    return int(_lib.lib().sa_forward_noalloc_read_status(_stream(stream)))


def read_device_status(workspace: torch.Tensor, stream=None) -> int:
    return int(_lib.lib().ska_read_device_status(_ptr(workspace), _stream(stream)))


def set_debug(wait_budget_ns: int = 0, flags: int = 0) -> None:
    _lib.lib().ska_set_debug(ctypes.c_uint64(wait_budget_ns), ctypes.c_uint32(flags))


def set_timing_events(start=None, stop=None) -> None:
    """Bench hook: record these torch.cuda.Events around the fused main kernel of later calls."""
    a = ctypes.c_void_p(start.cuda_event) if start is not None else ctypes.c_void_p(0)
    b = ctypes.c_void_p(stop.cuda_event) if stop is not None else ctypes.c_void_p(0)
    _lib.lib().ska_set_timing_events(a, b)


def stca_desc(q, k_hist, k_sk, cu_targets, cu_hist, *, scale, max_targets: int = 0) -> StcaDesc:
    d = StcaDesc()
    d.num_users = cu_targets.numel() - 1
    d.num_heads = q.shape[1]
    d.head_dim = q.shape[2]
    d.num_sketch = k_sk.shape[2] if k_sk is not None else 0
    d.total_targets = q.shape[0]
    d.total_hist = k_hist.shape[0] if k_hist is not None else 0
    d.max_targets = int(max_targets)
    d.max_hist = 0
    d.scale = float(scale)
    d.reserved = 0
    return d


def stca_forward_workspace_size(desc: StcaDesc) -> int:
    return int(_lib.lib().stca_forward_workspace_size(ctypes.byref(desc)))


def stca_forward(q: torch.Tensor, cu_targets: torch.Tensor, k_hist: torch.Tensor, v_hist: torch.Tensor,
                 cu_hist: torch.Tensor, k_sk: Optional[torch.Tensor], v_sk: Optional[torch.Tensor], *,
                 scale: float, target_kv_len: Optional[torch.Tensor] = None, want_lse: bool = True,
                 max_targets: Optional[int] = None, workspace: Optional[torch.Tensor] = None, stream=None,
                 out: Optional[torch.Tensor] = None, lse_out: Optional[torch.Tensor] = None):
    """STCA forward (SequenceO1 §2.3; the suffix and sketch branches of §3.4; MRLB §4.2).

    q [Tq,H,d] bf16 with cu_targets int32 [B+1]; k_hist, v_hist [Th,H,d] bf16 with cu_hist;
    k_sk, v_sk [B,H,ks,d] bf16 or None; target_kv_len int32 [Tq] or None; max_targets: an upper
    bound on any user's target count (read from cu_targets when None, which synchronises);
    out / lse_out: preallocated outputs (fp32 [Tq,H,d] / [Tq,H]). A max_targets below a user's
    real target count is recorded in the device status word and makes every output NaN.
    Returns (out fp32 [Tq,H,d], lse fp32 [Tq,H] or None).
    """
    for name, t in (("q", q), ("k_hist", k_hist), ("v_hist", v_hist), ("k_sk", k_sk), ("v_sk", v_sk)):
        if t is not None and t.dtype != torch.bfloat16:
            raise ValueError(f"{name} has dtype {t.dtype}, expected torch.bfloat16")
    if q.dim() != 3:
        raise ValueError(f"q must be [Tq, H, d], got shape {tuple(q.shape)}")
    Tq, H, D = q.shape
    for name, t in (("cu_targets", cu_targets), ("cu_hist", cu_hist)):
        if t.dtype != torch.int32 or t.dim() != 1 or t.numel() < 1:
            raise ValueError(f"{name} must be a 1-D int32 tensor of B + 1 offsets")
    B = cu_targets.numel() - 1
    if cu_hist.numel() != B + 1:
        raise ValueError(f"cu_hist has {cu_hist.numel()} entries, cu_targets {B + 1}")
    if k_hist is not None:
        if k_hist.dim() != 3 or k_hist.shape[1:] != (H, D):
            raise ValueError(f"k_hist {tuple(k_hist.shape)} does not match q's heads and head_dim")
        _shape("v_hist", v_hist, k_hist.shape)
    if (k_sk is None) != (v_sk is None):
        raise ValueError("k_sk and v_sk come together")
    if k_sk is not None:
        if k_sk.dim() != 4 or k_sk.shape[0] != B or k_sk.shape[1] != H or k_sk.shape[3] != D:
            raise ValueError(f"k_sk must be [{B}, {H}, ks, {D}], got {tuple(k_sk.shape)}")
        _shape("v_sk", v_sk, k_sk.shape)
    if target_kv_len is not None and (target_kv_len.dtype != torch.int32 or tuple(target_kv_len.shape) != (Tq,)):
        raise ValueError(f"target_kv_len must be int32 of shape ({Tq},)")
    _shape("out", out, (Tq, H, D))
    _shape("lse_out", lse_out, (Tq, H))
    if max_targets is None:
        max_targets = int((cu_targets[1:] - cu_targets[:-1]).max().item()) if cu_targets.numel() > 1 else 0
    for name, t in (("q", q), ("k_hist", k_hist), ("v_hist", v_hist), ("k_sk", k_sk), ("v_sk", v_sk)):
        _dev_tensor(name, t, (torch.bfloat16,))
    for name, t in (("cu_targets", cu_targets), ("cu_hist", cu_hist), ("target_kv_len", target_kv_len)):
        _dev_tensor(name, t, (torch.int32,))
    desc = stca_desc(q, k_hist, k_sk, cu_targets, cu_hist, scale=scale, max_targets=max(max_targets, 1))
    dev = q.device
    need = stca_forward_workspace_size(desc)
    if need == 0 and desc.total_targets > 0:
        raise SkaError(_lib.SKA_ERR_UNSUPPORTED, "stca_forward_workspace_size")
    if workspace is None or workspace.numel() < need:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=dev)
    out = torch.empty(q.shape, dtype=torch.float32, device=dev) if out is None else out
    if want_lse:
        lse = torch.empty(q.shape[:2], dtype=torch.float32, device=dev) if lse_out is None else lse_out
    else:
        lse = None
    _dev_tensor("out", out, (torch.float32,))
    _dev_tensor("lse_out", lse, (torch.float32,))
    rc = _lib.lib().stca_forward(ctypes.byref(desc), _ptr(q), _ptr(cu_targets), _ptr(k_hist), _ptr(v_hist),
                                 _ptr(cu_hist), _ptr(target_kv_len), _ptr(k_sk), _ptr(v_sk), _ptr(out),
                                 _ptr(lse), _ptr(workspace), ctypes.c_size_t(workspace.numel()), _stream(stream))
    _check(rc, "stca_forward")
    return out, lse


def stca_backward(q: torch.Tensor, cu_targets: torch.Tensor, k_hist: torch.Tensor, v_hist: torch.Tensor,
                  cu_hist: torch.Tensor, k_sk: Optional[torch.Tensor], v_sk: Optional[torch.Tensor],
                  out: torch.Tensor, lse: torch.Tensor, dout: torch.Tensor, *, scale: float,
                  target_kv_len: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
                  stream=None):
    """STCA backward (SequenceO1 §2.3, §3.4): gradients of <dout, out> through stca_forward.

    Inputs as in stca_forward, plus its outputs out fp32 [Tq,H,d] and lse fp32 [Tq,H], and dout
    bf16 [Tq,H,d]. Returns (dq [Tq,H,d], dk_hist, dv_hist [Th,H,d], dk_sk, dv_sk [B,H,ks,d] or
    None), all fp32.
    """
    for name, t in (("q", q), ("k_hist", k_hist), ("v_hist", v_hist), ("k_sk", k_sk), ("v_sk", v_sk),
                    ("dout", dout)):
        if t is not None and t.dtype != torch.bfloat16:
            raise ValueError(f"{name} has dtype {t.dtype}, expected torch.bfloat16")
    if q.dim() != 3:
        raise ValueError(f"q must be [Tq, H, d], got shape {tuple(q.shape)}")
    Tq, H, D = q.shape
    for name, t in (("cu_targets", cu_targets), ("cu_hist", cu_hist)):
        if t.dtype != torch.int32 or t.dim() != 1 or t.numel() < 1:
            raise ValueError(f"{name} must be a 1-D int32 tensor of B + 1 offsets")
    B = cu_targets.numel() - 1
    if cu_hist.numel() != B + 1:
        raise ValueError(f"cu_hist has {cu_hist.numel()} entries, cu_targets {B + 1}")
    if k_hist.dim() != 3 or k_hist.shape[1:] != (H, D):
        raise ValueError(f"k_hist {tuple(k_hist.shape)} does not match q's heads and head_dim")
    _shape("v_hist", v_hist, k_hist.shape)
    if (k_sk is None) != (v_sk is None):
        raise ValueError("k_sk and v_sk come together")
    if k_sk is not None:
        if k_sk.dim() != 4 or k_sk.shape[0] != B or k_sk.shape[1] != H or k_sk.shape[3] != D:
            raise ValueError(f"k_sk must be [{B}, {H}, ks, {D}], got {tuple(k_sk.shape)}")
        _shape("v_sk", v_sk, k_sk.shape)
    _shape("out", out, (Tq, H, D))
    _shape("lse", lse, (Tq, H))
    _shape("dout", dout, (Tq, H, D))
    if target_kv_len is not None and (target_kv_len.dtype != torch.int32 or tuple(target_kv_len.shape) != (Tq,)):
        raise ValueError(f"target_kv_len must be int32 of shape ({Tq},)")
    for name, t in (("q", q), ("k_hist", k_hist), ("v_hist", v_hist), ("k_sk", k_sk), ("v_sk", v_sk),
                    ("dout", dout)):
        _dev_tensor(name, t, (torch.bfloat16,))
    for name, t in (("out", out), ("lse", lse)):
        _dev_tensor(name, t, (torch.float32,))
    for name, t in (("cu_targets", cu_targets), ("cu_hist", cu_hist), ("target_kv_len", target_kv_len)):
        _dev_tensor(name, t, (torch.int32,))
    desc = stca_desc(q, k_hist, k_sk, cu_targets, cu_hist, scale=scale, max_targets=max(Tq, 1))
    L = _lib.lib()
    need = int(L.stca_backward_workspace_size(ctypes.byref(desc)))
    dev = q.device
    if workspace is None or workspace.numel() < need:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=dev)
    dq = torch.empty((Tq, H, D), dtype=torch.float32, device=dev)
    dkh = torch.empty(k_hist.shape, dtype=torch.float32, device=dev)
    dvh = torch.empty(k_hist.shape, dtype=torch.float32, device=dev)
    dks = torch.empty(k_sk.shape, dtype=torch.float32, device=dev) if k_sk is not None else None
    dvs = torch.empty(k_sk.shape, dtype=torch.float32, device=dev) if k_sk is not None else None
    rc = L.stca_backward(ctypes.byref(desc), _ptr(q), _ptr(cu_targets), _ptr(k_hist), _ptr(v_hist), _ptr(cu_hist),
                         _ptr(target_kv_len), _ptr(k_sk), _ptr(v_sk), _ptr(out), _ptr(lse), _ptr(dout), _ptr(dq),
                         _ptr(dkh), _ptr(dvh), _ptr(dks), _ptr(dvs), _ptr(workspace),
                         ctypes.c_size_t(workspace.numel()), _stream(stream))
    _check(rc, "stca_backward")
    return dq, dkh, dvh, dks, dvs


def sa_backward_workspace_size(desc: SaDesc) -> int:
    return int(_lib.lib().sa_backward_workspace_size(ctypes.byref(desc)))


def sa_backward(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, cu_seqlens: torch.Tensor,
                seqused: Optional[torch.Tensor], lse: torch.Tensor, dsketch: torch.Tensor,
                sketch: Optional[torch.Tensor] = None, *, scale: float = 1.0, norm="proto",
                workspace: Optional[torch.Tensor] = None, stream=None, outs=None):
    """SA backward (gradients of <dsketch, sketch> through SequenceO1 §3.1 Eq. (7)-(9)).

    bf16 q, k, v, dsketch; the forward's lse (and, for norm="token", its sketch); outs: an
    optional preallocated (dq, dk, dv).
    Returns (dq fp32 shaped like q, dk fp32 [T,H,d], dv fp32 [T,H,d]).
    """
    B, H, kp, D = _check_sa_inputs(q, k, v, cu_seqlens, seqused, (torch.bfloat16,))
    nid = _NORMS[norm]
    if dsketch.dtype != torch.bfloat16:
        raise ValueError(f"dsketch has dtype {dsketch.dtype}, expected torch.bfloat16")
    _shape("dsketch", dsketch, (B, H, kp, D))
    if lse.dtype != torch.float32:
        raise ValueError(f"lse has dtype {lse.dtype}, expected torch.float32")
    _shape("lse", lse, (k.shape[0], H) if nid == _lib.SKA_NORM_PROTO else (B, H, kp))
    if nid == _lib.SKA_NORM_TOKEN and sketch is None:
        raise ValueError("the token-wise backward needs the forward sketch (D_j = dO_j . O_j)")
    if sketch is not None and sketch.dtype != torch.float32:
        raise ValueError(f"sketch has dtype {sketch.dtype}, expected torch.float32")
    _shape("sketch", sketch, (B, H, kp, D))
    for name, t in (("q", q), ("k", k), ("v", v), ("dsketch", dsketch)):
        _dev_tensor(name, t, (torch.bfloat16,))
    _dev_tensor("lse", lse, (torch.float32,))
    _dev_tensor("sketch", sketch, (torch.float32,))
    _dev_tensor("cu_seqlens", cu_seqlens, (torch.int32,))
    _dev_tensor("seqused", seqused, (torch.int32,))
    desc = sa_desc(q, k, cu_seqlens, scale=scale, norm=norm)
    dev = k.device
    need = sa_backward_workspace_size(desc)
    if need == 0:
        raise SkaError(_lib.SKA_ERR_UNSUPPORTED, "sa_backward_workspace_size")
    if workspace is None or workspace.numel() < need:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    if outs is None:
        outs = (torch.empty(q.shape, dtype=torch.float32, device=dev), torch.empty(k.shape, dtype=torch.float32,
                device=dev), torch.empty(v.shape, dtype=torch.float32, device=dev))
    dq, dk, dv = outs
    for name, t, like in (("dq", dq, q), ("dk", dk, k), ("dv", dv, v)):
        _dev_tensor(name, t, (torch.float32,))
        if t.shape != like.shape:
            raise ValueError(f"{name}: shape {tuple(t.shape)}, expected {tuple(like.shape)}")
    rc = _lib.lib().sa_backward(ctypes.byref(desc), _ptr(q), _ptr(k), _ptr(v), _ptr(cu_seqlens), _ptr(seqused),
                                _ptr(sketch), _ptr(lse), _ptr(dsketch), _ptr(dq), _ptr(dk), _ptr(dv),
                                _ptr(workspace), ctypes.c_size_t(workspace.numel()), _stream(stream))
    _check(rc, "sa_backward")
    return dq, dk, dv


def refine_desc(x_tilde, x_hat, w1, *, eps: float = 1e-5) -> RefineDesc:
    d = RefineDesc()
    d.num_users, d.num_heads, d.num_protos, d.head_dim = (int(v) for v in x_hat.shape)
    d.ffn_dim = int(w1.shape[-1])
    d.eps = float(eps)
    d.x_tilde_shared = 1 if x_tilde.dim() == 3 else 0
    d.reserved = 0
    return d


def sa_refine_workspace_size(desc: RefineDesc) -> int:
    return int(_lib.lib().sa_refine_workspace_size(ctypes.byref(desc)))


def sa_refine(x_tilde: torch.Tensor, x_hat: torch.Tensor, w1: torch.Tensor, wg: torch.Tensor, w2: torch.Tensor,
              gamma1: Optional[torch.Tensor] = None, beta1: Optional[torch.Tensor] = None,
              gamma2: Optional[torch.Tensor] = None, beta2: Optional[torch.Tensor] = None, *, eps: float = 1e-5,
              w_q_next: Optional[torch.Tensor] = None, want_x_bar: bool = False, want_bf16: bool = False,
              workspace: Optional[torch.Tensor] = None, out: Optional[torch.Tensor] = None, stream=None):
    """Stacked refinement of the sketch (SequenceO1 §3.3, Eq. (13)-(14)) with the SwiGLU FFN of
    App. G.1: x_bar = LN1(x_tilde + x_hat), x_next = LN2(x_bar + (swish(x_bar W1) * (x_bar Wg)) W2).

    x_hat fp32 [B,H,k,d] (this layer's sa_forward sketch); x_tilde fp32 [B,H,k,d], or [H,k,d] for
    rows shared by every user (layer 0: the prototypes); w1, wg bf16 [H,d,F]; w2 bf16 [H,F,d] with
    F = 2d; gamma*, beta* fp32 [H,d] or None; w_q_next bf16 [H,d,d] or None: also return the next
    layer's per-user queries x_next W_Q (Eq. (10)). Returns (x_next fp32, x_bar fp32 or None,
    x_next bf16 or None, q_next bf16 or None), each [B,H,k,d].
    """
    if x_hat.dim() != 4:
        raise ValueError(f"x_hat must be [B, H, k, d], got shape {tuple(x_hat.shape)}")
    B, H, k, D = x_hat.shape
    if x_tilde.dim() == 3:
        _shape("x_tilde", x_tilde, (H, k, D))
    else:
        _shape("x_tilde", x_tilde, x_hat.shape)
    if w1.dim() != 3 or w1.shape[0] != H or w1.shape[1] != D:
        raise ValueError(f"w1 must be [{H}, {D}, F], got {tuple(w1.shape)}")
    F = w1.shape[2]
    _shape("wg", wg, (H, D, F))
    _shape("w2", w2, (H, F, D))
    _shape("w_q_next", w_q_next, (H, D, D))
    for name, t in (("gamma1", gamma1), ("beta1", beta1), ("gamma2", gamma2), ("beta2", beta2)):
        _shape(name, t, (H, D))
    _shape("out", out, x_hat.shape)
    acts = (("x_tilde", x_tilde), ("x_hat", x_hat), ("gamma1", gamma1), ("beta1", beta1), ("gamma2", gamma2),
            ("beta2", beta2), ("out", out))
    weights = (("w1", w1), ("wg", wg), ("w2", w2), ("w_q_next", w_q_next))
    _dtypes(acts, (torch.float32,))
    _dtypes(weights, (torch.bfloat16,))
    for name, t in acts:
        _dev_tensor(name, t, (torch.float32,))
    for name, t in weights:
        _dev_tensor(name, t, (torch.bfloat16,))
    desc = refine_desc(x_tilde, x_hat, w1, eps=eps)
    L = _lib.lib()
    need = sa_refine_workspace_size(desc)
    if need == 0:
        _check(L.sa_refine(ctypes.byref(desc), *([ctypes.c_void_p(0)] * 15), ctypes.c_size_t(0),
                           ctypes.c_void_p(0)), "sa_refine")
    dev = x_hat.device
    if workspace is None or workspace.numel() < need:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=dev)
    out = torch.empty(x_hat.shape, dtype=torch.float32, device=dev) if out is None else out
    x_bar = torch.empty(x_hat.shape, dtype=torch.float32, device=dev) if want_x_bar else None
    x_bf = torch.empty(x_hat.shape, dtype=torch.bfloat16, device=dev) if want_bf16 else None
    q_next = torch.empty(x_hat.shape, dtype=torch.bfloat16, device=dev) if w_q_next is not None else None
    rc = L.sa_refine(ctypes.byref(desc), _ptr(x_tilde), _ptr(x_hat), _ptr(w1), _ptr(wg), _ptr(w2), _ptr(gamma1),
                     _ptr(beta1), _ptr(gamma2), _ptr(beta2), _ptr(w_q_next), _ptr(out), _ptr(x_bar), _ptr(x_bf),
                     _ptr(q_next), _ptr(workspace), ctypes.c_size_t(workspace.numel()), _stream(stream))
    _check(rc, "sa_refine")
    return out, x_bar, x_bf, q_next


def project_queries(x: torch.Tensor, w_q: torch.Tensor, *, workspace: Optional[torch.Tensor] = None,
                    out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """q = x W_Q for each head (SequenceO1 Eq. (7) P^(0) W_Q; Eq. (10) X~^(l) W_Q^(l)).

    x fp32 [H,k,d] (the prototypes) or [B,H,k,d]; w_q bf16 [H,d,d]. Returns q bf16 of x's shape.
    """
    if x.dim() not in (3, 4):
        raise ValueError(f"x must be [H, k, d] or [B, H, k, d], got shape {tuple(x.shape)}")
    shape4 = (1,) + tuple(x.shape) if x.dim() == 3 else tuple(x.shape)
    B, H, k, D = shape4
    _shape("w_q", w_q, (H, D, D))
    _shape("out", out, x.shape)
    _dtypes((("x", x),), (torch.float32,))
    _dtypes((("w_q", w_q), ("out", out)), (torch.bfloat16,))
    _dev_tensor("x", x, (torch.float32,))
    _dev_tensor("w_q", w_q, (torch.bfloat16,))
    _dev_tensor("out", out, (torch.bfloat16,))
    if workspace is None or workspace.numel() < 256:
        workspace = torch.empty(256, dtype=torch.uint8, device=x.device)
    out = torch.empty(x.shape, dtype=torch.bfloat16, device=x.device) if out is None else out
    rc = _lib.lib().sa_project_queries(B, H, k, D, _ptr(x), _ptr(w_q), _ptr(out), _ptr(workspace),
                                       ctypes.c_size_t(workspace.numel()), _stream(stream))
    _check(rc, "sa_project_queries")
    return out


def cache_keys(user_id, model_version, sketch_config, history_timestamp, device="cuda") -> torch.Tensor:
    """Keys of the sketch cache as the C ABI lays them out (ska_cache_key, 24 bytes): an int64
    tensor [n, 3] holding the user id, the version in the low and the configuration in the high
    32 bits, and the history timestamp."""
    u = torch.as_tensor(user_id, dtype=torch.int64).reshape(-1)
    v = torch.as_tensor(model_version, dtype=torch.int64).reshape(-1) & 0xFFFFFFFF
    c = torch.as_tensor(sketch_config, dtype=torch.int64).reshape(-1) & 0xFFFFFFFF
    t = torch.as_tensor(history_timestamp, dtype=torch.int64).reshape(-1)
    n = max(u.numel(), v.numel(), c.numel(), t.numel())
    word1 = v.expand(n) | (c.expand(n) << 32)
    return torch.stack([u.expand(n), word1, t.expand(n)], dim=1).contiguous().to(device)


class SketchCache:
    """Device-side sketch cache of SequenceO1 §4.1 (see sa_cache_* in include/sketch_attn.h):
    num_sets sets x ways ways of rows of row_floats floats, entries live for ttl time units."""

    def __init__(self, num_sets: int, ways: int, row_floats: int, ttl: int, device="cuda", stream=None):
        from ._lib import CacheDesc
        self.desc = CacheDesc(num_sets, ways, row_floats, 0, ttl)
        L = _lib.lib()
        nbytes = int(L.sa_cache_bytes(ctypes.byref(self.desc)))
        if nbytes == 0:
            raise SkaError(_lib.SKA_ERR_INVALID_VALUE, "sa_cache_bytes")
        self.mem = torch.empty(nbytes, dtype=torch.uint8, device=device)
        self.row_floats = row_floats
        _check(L.sa_cache_init(ctypes.byref(self.desc), _ptr(self.mem), ctypes.c_size_t(nbytes), _stream(stream)),
               "sa_cache_init")

    def put(self, keys: torch.Tensor, rows: torch.Tensor, now: int, stream=None) -> torch.Tensor:
        if keys.dim() != 2 or keys.shape[1] != 3 or keys.dtype != torch.int64:
            raise ValueError("keys must be an int64 [n, 3] tensor (see cache_keys)")
        n = keys.shape[0]
        _shape("rows", rows, (n, self.row_floats))
        _dev_tensor("keys", keys, (torch.int64,))
        _dev_tensor("rows", rows, (torch.float32,))
        slots = torch.empty(n, dtype=torch.int32, device=keys.device)
        _check(_lib.lib().sa_cache_put(ctypes.byref(self.desc), _ptr(self.mem), ctypes.c_size_t(self.mem.numel()),
                                       _ptr(keys), _ptr(rows), n, int(now), _ptr(slots), _stream(stream)),
               "sa_cache_put")
        return slots

    def get(self, keys: torch.Tensor, now: int, stream=None):
        if keys.dim() != 2 or keys.shape[1] != 3 or keys.dtype != torch.int64:
            raise ValueError("keys must be an int64 [n, 3] tensor (see cache_keys)")
        _dev_tensor("keys", keys, (torch.int64,))
        n = keys.shape[0]
        out = torch.empty((n, self.row_floats), dtype=torch.float32, device=keys.device)
        hits = torch.empty(n, dtype=torch.int32, device=keys.device)
        _check(_lib.lib().sa_cache_get(ctypes.byref(self.desc), _ptr(self.mem), ctypes.c_size_t(self.mem.numel()),
                                       _ptr(keys), n, int(now), _ptr(out), _ptr(hits), _stream(stream)),
               "sa_cache_get")
        return out, hits
