"""B200 (sm_100a) block-sparse attention: cumulative-energy block mask + sparse forward.

Thin binding over the C ABI (include/sparse_attn.h): every call below only checks
and marshals torch tensors into pointers and sizes, then calls the library, which
runs all the work in its CUDA kernels on the tensors' device and the current
torch stream. PyTorch provides device memory and streams, nothing else.

    plan = sparse_attn_plan(q, k, tau=0.95)            # stage 1: block mask
    o = sparse_attn_fwd(q, k, v, plan, lam=-12.0)      # stage 2: sparse attention

q, k, v: bf16 CUDA tensors [B, H, N, d], contiguous, d in {64, 128}.
"""
from __future__ import annotations

import ctypes
import math
from dataclasses import dataclass
from typing import Optional, Union

import torch

from . import _lib
from ._lib import SaShape, SparseAttnError

BLOCK = 64

__all__ = ["Plan", "sparse_attn_plan", "sparse_attn_fwd", "sparse_attn_fwd_recall", "sparse_attention",
           "Clustering", "sparse_attn_cluster", "sparse_attn_cluster_workspace_size", "sparse_attn_permute_rows",
           "sparse_attention_clustered",
           "sparse_attn_plan_workspace_size", "sparse_attn_num_tiles", "sparse_attn_device_error",
           "sparse_attn_host_workspace_size",
           "sparse_attn_selftest_wait_timeout",
           "SparseAttnError", "BLOCK"]


def _shape(q: torch.Tensor) -> SaShape:
    B, H, N, d = q.shape
    return SaShape(B, H, N, d, BLOCK)


def _check_qkv(*ts: torch.Tensor):
    q = ts[0]
    for t in ts:
        if not t.is_cuda:
            raise ValueError("tensors must be CUDA tensors")
        if t.dtype != torch.bfloat16:
            raise ValueError("tensors must be bf16")
        if t.dim() != 4 or t.shape != q.shape:
            raise ValueError("q, k, v must share the shape [B, H, N, d]")
        if not t.is_contiguous():
            raise ValueError("tensors must be contiguous [B, H, N, d]")
        if t.device != q.device:
            raise ValueError("tensors must be on one device")


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(device) -> ctypes.c_void_p:
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _call(name: str, status: int):
    if status != _lib.SA_OK:
        raise SparseAttnError(name, status, _lib.load())


@dataclass
class Plan:
    """Output of sparse_attn_plan (all on the inputs' device).

    mask  uint8 [B, H, Nb, Nb]  1 = kept key block
    count int32 [B, H, Nb]      kept blocks per query block
    idx   int32 [B, H, Nb, Nb]  ascending kept blocks in the first count entries
                                of each row (rest of the row undefined), or None
    work  int32 [2*num_tiles]   query-block pairs in execution order for sparse_attn_fwd
                                (global ids (b*H+h)*Nb+i, second -1 if absent), or None
    q8, k8          uint8 [B, H, N, d]  8-bit codes of q and k (quantize="fp8": FP8 E4M3;
                                        quantize="int8": int8 values), else None
    qscale, kscale  float32 [B, H, Nb]  their per-block scales, else None
    qfmt            "fp8", "int8" or None: the format of q8 and k8
    """
    mask: torch.Tensor
    count: torch.Tensor
    idx: Optional[torch.Tensor]
    work: Optional[torch.Tensor]
    tau: Union[float, torch.Tensor]   # one threshold, or one per (batch, head)
    causal: bool
    qfmt: Optional[str] = None
    q8: Optional[torch.Tensor] = None
    k8: Optional[torch.Tensor] = None
    qscale: Optional[torch.Tensor] = None
    kscale: Optional[torch.Tensor] = None


def sparse_attn_plan_workspace_size(B: int, H: int, N: int, d: int) -> int:
    return int(_lib.load().sparse_attn_plan_workspace_size(SaShape(B, H, N, d, BLOCK)))


def sparse_attn_num_tiles(B: int, H: int, N: int, d: int) -> int:
    return int(_lib.load().sparse_attn_num_tiles(SaShape(B, H, N, d, BLOCK)))


def sparse_attn_host_workspace_size(B: int, H: int, N: int, d: int, chunks: int = 4, qk_fp8: bool = False,
                                    qk_int8: bool = False) -> int:
    flags = (_lib.SA_HOST_FP8_SCORES if qk_fp8 else 0) | (_lib.SA_HOST_INT8_SCORES if qk_int8 else 0)
    return int(_lib.load().sparse_attn_host_workspace_size(SaShape(B, H, N, d, BLOCK), int(chunks), flags))


def sparse_attn_plan(q: torch.Tensor, k: torch.Tensor, tau, scale: Optional[float] = None,
                     causal: bool = False, *, with_idx: bool = False, with_work: bool = True,
                     out: Optional[Plan] = None, workspace: Optional[torch.Tensor] = None,
                     quantize=False) -> Plan:
    """Stage 1: cumulative-energy block mask from mean-pooled q and k.

    tau is one recall threshold for every head (a float), or one per head: a float32
    CUDA tensor of shape [B, H] or [H] on q's device (sparse_attn_plan_heads).
    quantize="fp8" (or True; one tau, d = 128) also writes FP8 E4M3 copies of q and k
    with per-block scales (sparse_attn_plan_q8) for sparse_attn_fwd(..., qk_fp8=True);
    quantize="int8" writes INT8 copies (sparse_attn_plan_i8) for qk_int8=True.
    with_idx=True also writes the ascending kept lists (an int32 [B, H, Nb, Nb]
    tensor: 4 bytes per block pair, 331 MB on the 118,800-token video shape); the
    forward does not read them, so they are off by default."""
    lib = _lib.load()
    _check_qkv(q, k)
    B, H, N, d = q.shape
    Nb = -(-N // BLOCK)
    s = _shape(q)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    dev = q.device
    if out is None:
        out = Plan(
            mask=torch.empty((B, H, Nb, Nb), dtype=torch.uint8, device=dev),
            count=torch.empty((B, H, Nb), dtype=torch.int32, device=dev),
            idx=torch.empty((B, H, Nb, Nb), dtype=torch.int32, device=dev) if with_idx else None,
            work=torch.empty((max(2, 2 * lib.sparse_attn_num_tiles(s)),), dtype=torch.int32, device=dev)
            if with_work else None,
            tau=tau if isinstance(tau, torch.Tensor) else float(tau), causal=bool(causal))
    else:
        out.tau, out.causal = (tau if isinstance(tau, torch.Tensor) else float(tau)), bool(causal)
    if quantize is True:
        quantize = "fp8"
    if quantize not in (False, None, "fp8", "int8"):
        raise ValueError('quantize must be False, True, "fp8" or "int8"')
    if quantize and out.q8 is None:
        out.q8 = torch.empty((B, H, N, d), dtype=torch.uint8, device=dev)
        out.k8 = torch.empty((B, H, N, d), dtype=torch.uint8, device=dev)
        out.qscale = torch.empty((B, H, Nb), dtype=torch.float32, device=dev)
        out.kscale = torch.empty((B, H, Nb), dtype=torch.float32, device=dev)
    ws_bytes = int(lib.sparse_attn_plan_workspace_size(s))
    if workspace is None or workspace.numel() < ws_bytes:
        workspace = torch.empty((max(ws_bytes, 256),), dtype=torch.uint8, device=dev)
    if quantize:
        if isinstance(tau, torch.Tensor):
            raise ValueError("quantize takes one tau for every head")
        fn = lib.sparse_attn_plan_i8 if quantize == "int8" else lib.sparse_attn_plan_q8
        st = fn(_ptr(q), _ptr(k), s, float(tau), float(scale), int(bool(causal)),
                _ptr(out.mask), _ptr(out.count), _ptr(out.idx), _ptr(out.work),
                _ptr(out.q8), _ptr(out.k8), _ptr(out.qscale), _ptr(out.kscale),
                _ptr(workspace), ws_bytes, _stream(dev))
        out.qfmt = quantize
        _call("sparse_attn_plan_i8" if quantize == "int8" else "sparse_attn_plan_q8", st)
        return out
    if isinstance(tau, torch.Tensor):
        if tau.dtype != torch.float32 or tau.device != dev:
            raise ValueError("a per-head tau must be a float32 tensor on q's device")
        if tuple(tau.shape) == (H,):
            tau = tau.unsqueeze(0).expand(B, H)
        if tuple(tau.shape) != (B, H):
            raise ValueError("a per-head tau must have shape [B, H] or [H]")
        tau = tau.contiguous()
        st = lib.sparse_attn_plan_heads(_ptr(q), _ptr(k), s, _ptr(tau), float(scale), int(bool(causal)),
                                        _ptr(out.mask), _ptr(out.count), _ptr(out.idx), _ptr(out.work),
                                        _ptr(workspace), ws_bytes, _stream(dev))
        _call("sparse_attn_plan_heads", st)
        return out
    st = lib.sparse_attn_plan(_ptr(q), _ptr(k), s, float(tau), float(scale), int(bool(causal)),
                              _ptr(out.mask), _ptr(out.count), _ptr(out.idx), _ptr(out.work),
                              _ptr(workspace), ws_bytes, _stream(dev))
    _call("sparse_attn_plan", st)
    return out


def sparse_attn_fwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, plan, lam: Optional[float] = None,
                    scale: Optional[float] = None, causal: Optional[bool] = None, *,
                    out: Optional[torch.Tensor] = None, stats: Optional[torch.Tensor] = None,
                    qk_fp8: bool = False, recall: Optional[float] = None,
                    decisions: Optional[torch.Tensor] = None, qk_int8: bool = False) -> torch.Tensor:
    """Stage 2: attention over the kept blocks with the lambda P.V filter.

    `plan` is a Plan or a uint8 mask [B, H, Nb, Nb]. lam=None turns the filter off.
    `stats`, if given, is an int64 CUDA tensor of 4 entries (see the C header).
    qk_fp8=True takes the scores on the plan's FP8 copies of q and k
    (sparse_attn_fwd_q8; the plan must come from sparse_attn_plan(quantize="fp8")),
    qk_int8=True on its INT8 copies (sparse_attn_fwd_i8; quantize="int8").
    recall=rho (in (0, 1]) replaces the lambda test by the cumulative-energy test
    of sparse_attn_fwd_recall: every row keeps at least the fraction rho of the
    softmax energy of the blocks it visits; lam must then be None.
    decisions, if given (uint8 [B, H, Nb, Nb] on q's device, bf16 scores), receives
    the filter's per-pair decisions (sparse_attn_fwd_decisions): 1 where a visited
    pair's P.V was skipped, 0 where it was computed; other entries are untouched."""
    lib = _lib.load()
    _check_qkv(q, k, v)
    B, H, N, d = q.shape
    Nb = -(-N // BLOCK)
    if isinstance(plan, Plan):
        mask, work = plan.mask, plan.work
        if causal is None:
            causal = plan.causal
    else:
        mask, work = plan, None
    causal = bool(causal)
    if mask.dtype != torch.uint8 or tuple(mask.shape) != (B, H, Nb, Nb) or not mask.is_contiguous() \
            or mask.device != q.device:
        raise ValueError("mask must be a contiguous uint8 tensor [B, H, Nb, Nb] on q's device")
    if work is not None and (work.dtype != torch.int32 or work.device != q.device):
        raise ValueError("work must be int32 on q's device")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    lam_f = -math.inf if lam is None else float(lam)
    if out is None:
        out = torch.empty_like(q)
    if stats is not None and (stats.dtype != torch.int64 or stats.numel() < 4 or stats.device != q.device):
        raise ValueError("stats must be an int64 tensor of >= 4 entries on q's device")
    if decisions is not None:
        if qk_fp8 or qk_int8:
            raise ValueError("decisions are recorded by the bf16-score forward")
        if decisions.dtype != torch.uint8 or tuple(decisions.shape) != (B, H, Nb, Nb) \
                or not decisions.is_contiguous() or decisions.device != q.device:
            raise ValueError("decisions must be a contiguous uint8 tensor [B, H, Nb, Nb] on q's device")
        if recall is not None and lam is not None:
            raise ValueError("recall replaces the lambda filter: pass lam=None with it")
        filt, val = (_lib.SA_FILTER_RECALL, float(recall)) if recall is not None else (_lib.SA_FILTER_LAMBDA, lam_f)
        st = lib.sparse_attn_fwd_decisions(_ptr(q), _ptr(k), _ptr(v), _shape(q), _ptr(mask), _ptr(work), filt, val,
                                           float(scale), int(causal), _ptr(out), _ptr(stats), _ptr(decisions),
                                           _stream(q.device))
        _call("sparse_attn_fwd_decisions", st)
        return out
    if recall is not None:
        if lam is not None or qk_fp8 or qk_int8:
            raise ValueError("recall replaces the lambda filter and takes bf16 scores: "
                             "pass lam=None and qk_fp8=False with it")
        st = lib.sparse_attn_fwd_recall(_ptr(q), _ptr(k), _ptr(v), _shape(q), _ptr(mask), _ptr(work),
                                        float(recall), float(scale), int(causal), _ptr(out), _ptr(stats),
                                        _stream(q.device))
        _call("sparse_attn_fwd_recall", st)
        return out
    if qk_fp8 or qk_int8:
        want = "int8" if qk_int8 else "fp8"
        if qk_fp8 and qk_int8:
            raise ValueError("qk_fp8 and qk_int8 exclude each other")
        if not isinstance(plan, Plan) or plan.q8 is None or plan.qfmt != want:
            raise ValueError(f'qk_{want}=True needs a plan made with quantize="{want}"')
        fn = lib.sparse_attn_fwd_i8 if qk_int8 else lib.sparse_attn_fwd_q8
        st = fn(_ptr(plan.q8), _ptr(plan.k8), _ptr(plan.qscale), _ptr(plan.kscale), _ptr(v),
                                    _shape(q), _ptr(mask), _ptr(work), lam_f, float(scale), int(causal),
                                    _ptr(out), _ptr(stats), _stream(q.device))
        _call("sparse_attn_fwd_i8" if qk_int8 else "sparse_attn_fwd_q8", st)
        return out
    st = lib.sparse_attn_fwd(_ptr(q), _ptr(k), _ptr(v), _shape(q), _ptr(mask), _ptr(work), lam_f,
                             float(scale), int(causal), _ptr(out), _ptr(stats), _stream(q.device))
    _call("sparse_attn_fwd", st)
    return out


def sparse_attn_fwd_recall(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, plan, recall: float,
                           scale: Optional[float] = None, causal: Optional[bool] = None, *,
                           out: Optional[torch.Tensor] = None,
                           stats: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Stage 2 with the cumulative-energy P.V filter (the C call of the same name):
    sparse_attn_fwd(q, k, v, plan, None, scale, causal, recall=recall, ...)."""
    return sparse_attn_fwd(q, k, v, plan, None, scale, causal, out=out, stats=stats, recall=recall)


@dataclass
class Clustering:
    """Output of sparse_attn_cluster (on the inputs' device).

    perm      int32 [B, H, N]     perm[b, h, p] = the token at position p in cluster order
    assign    int32 [B, H, N]     each token's cluster, or None
    centroids fp32 [B, H, C, d]   the final cluster means (C = ceil(N/64)), or None
    """
    perm: torch.Tensor
    assign: Optional[torch.Tensor] = None
    centroids: Optional[torch.Tensor] = None


def sparse_attn_cluster_workspace_size(B: int, H: int, N: int, d: int) -> int:
    return int(_lib.load().sparse_attn_cluster_workspace_size(SaShape(B, H, N, d, BLOCK)))


def sparse_attn_cluster(x: torch.Tensor, y: torch.Tensor, iters: int = 2, *, with_assign: bool = True,
                        with_centroids: bool = False, out: Optional[Clustering] = None,
                        workspace: Optional[torch.Tensor] = None) -> Clustering:
    """Interaction clustering of x's tokens under the Gram metric of y (the C call
    of the same name): queries are clustered with y = k, keys with y = q."""
    lib = _lib.load()
    _check_qkv(x, y)
    B, H, N, d = x.shape
    C = -(-N // BLOCK)
    dev = x.device
    if out is None:
        out = Clustering(
            perm=torch.empty((B, H, N), dtype=torch.int32, device=dev),
            assign=torch.empty((B, H, N), dtype=torch.int32, device=dev) if with_assign else None,
            centroids=torch.empty((B, H, C, d), dtype=torch.float32, device=dev) if with_centroids else None)
    if workspace is None:
        workspace = torch.empty(sparse_attn_cluster_workspace_size(B, H, N, d), dtype=torch.uint8, device=dev)
    st = lib.sparse_attn_cluster(_ptr(x), _ptr(y), _shape(x), int(iters), _ptr(out.assign), _ptr(out.perm),
                                 _ptr(out.centroids), _ptr(workspace), workspace.numel(), _stream(dev))
    _call("sparse_attn_cluster", st)
    return out


def sparse_attn_permute_rows(src: torch.Tensor, perm: torch.Tensor, inverse: bool = False, *,
                             out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Rows of src [B, H, N, d] moved by perm [B, H, N] (int32): gathered
    (out[b, h, p] = src[b, h, perm[b, h, p]]) or, with inverse, scattered."""
    lib = _lib.load()
    _check_qkv(src)
    if perm.dtype != torch.int32 or tuple(perm.shape) != tuple(src.shape[:3]) or perm.device != src.device \
            or not perm.is_contiguous():
        raise ValueError("perm must be a contiguous int32 tensor [B, H, N] on src's device")
    if out is None:
        out = torch.empty_like(src)
    st = lib.sparse_attn_permute_rows(_ptr(src), _ptr(perm), _shape(src), int(bool(inverse)), _ptr(out),
                                      _stream(src.device))
    _call("sparse_attn_permute_rows", st)
    return out


def sparse_attention_clustered(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, tau, lam: Optional[float] = None,
                               iters: int = 2, scale: Optional[float] = None, *,
                               recall: Optional[float] = None):
    """Plan + forward on tokens reordered by interaction clustering (non-causal):
    queries clustered under k's Gram metric, keys under q's; q, k, v reordered,
    sparse_attn_plan and sparse_attn_fwd on the reordered tensors, and the output
    rows put back in token order. Returns (o, info) with info = dict(cq, ck, plan)."""
    _check_qkv(q, k, v)
    cq = sparse_attn_cluster(q, k, iters, with_assign=False)
    ck = sparse_attn_cluster(k, q, iters, with_assign=False)
    qs = sparse_attn_permute_rows(q, cq.perm)
    ks = sparse_attn_permute_rows(k, ck.perm)
    vs = sparse_attn_permute_rows(v, ck.perm)
    plan = sparse_attn_plan(qs, ks, tau, scale, False)
    os_ = sparse_attn_fwd(qs, ks, vs, plan, lam, scale, False, recall=recall)
    o = sparse_attn_permute_rows(os_, cq.perm, inverse=True)
    return o, dict(cq=cq, ck=ck, plan=plan)


_COPY_STREAMS = {}


def _copy_streams(dev: torch.device):
    """The two copy streams of `sparse_attention` on a device (host-to-device and
    device-to-host), created once per device and reused by every call."""
    idx = dev.index if dev.index is not None else torch.cuda.current_device()
    if idx not in _COPY_STREAMS:
        _COPY_STREAMS[idx] = (torch.cuda.Stream(idx), torch.cuda.Stream(idx))
    return _COPY_STREAMS[idx]


def sparse_attention(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, tau,
                     lam: Optional[float] = None, scale: Optional[float] = None, causal: bool = False,
                     device="cuda", out: Optional[torch.Tensor] = None, chunks: Optional[int] = None,
                     qk_fp8: bool = False, recall: Optional[float] = None,
                     workspace: Optional[torch.Tensor] = None, qk_int8: bool = False) -> torch.Tensor:
    """End to end from host tensors (the C call sparse_attn_host): copy q, k, v to
    the GPU, plan + forward, copy O back.

    Host inputs should be pinned, so the copies are asynchronous DMA. The result is
    a host bf16 tensor in pinned memory (`out` if given, else one from torch's
    caching pinned allocator), ready when this returns.

    Heads are independent, so the call is pipelined over `chunks` groups of heads
    (default: up to 4): group g's host-to-device copy, its plan + forward and its
    device-to-host copy run on three streams, so the copies of one group overlap
    the work of the others in both directions of the link. tau may be one value or
    a per-head float32 tensor ([B, H] or [H]) on `device`; qk_fp8=True takes the scores on FP8 copies of q and k (see
    sparse_attn_plan's quantize), qk_int8=True on INT8 copies; recall selects the cumulative-energy P.V filter
    instead of lambda (see sparse_attn_fwd). The device workspace is allocated
    here unless given (sparse_attn_host_workspace_size bytes).

    After the call the device error word is read: a device-side check that fired
    (a bounded wait that gave up, a range check) raises SparseAttnError with
    SA_ERR_DEVICE_CHECK, since O is then undefined for the affected rows."""
    lib = _lib.load()
    dev = torch.device(device)
    if dev.type == "cuda" and dev.index is None:
        dev = torch.device("cuda", torch.cuda.current_device())
    if q.shape != k.shape or q.shape != v.shape or q.dim() != 4:
        raise ValueError("q, k, v must share the shape [B, H, N, d]")
    for t in (q, k, v):
        if t.device.type != "cpu" or t.dtype != torch.bfloat16 or not t.is_contiguous():
            raise ValueError("q, k, v must be contiguous host bf16 tensors")
    if recall is not None and (lam is not None or qk_fp8 or qk_int8):
        raise ValueError("recall replaces the lambda filter and takes bf16 scores")
    B, H, N, d = q.shape
    if out is None:
        out = torch.empty(q.shape, dtype=q.dtype, pin_memory=True)
    elif out.shape != q.shape or out.dtype != q.dtype or out.device.type != "cpu" or not out.is_contiguous():
        raise ValueError("out must be a contiguous host bf16 tensor of q's shape")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    nch = max(1, min(B * H, chunks if chunks is not None else 4))
    if qk_fp8 and qk_int8:
        raise ValueError("qk_fp8 and qk_int8 exclude each other")
    flags = (_lib.SA_HOST_FP8_SCORES if qk_fp8 else 0) | (_lib.SA_HOST_INT8_SCORES if qk_int8 else 0)
    s = _shape(q)
    ws_bytes = int(lib.sparse_attn_host_workspace_size(s, nch, flags))
    if ws_bytes == 0:
        raise ValueError("unsupported shape for sparse_attention")
    if workspace is None or workspace.numel() < ws_bytes or workspace.device != dev:
        workspace = torch.empty((ws_bytes,), dtype=torch.uint8, device=dev)
    tau_heads = None
    if isinstance(tau, torch.Tensor):
        if tau.dtype != torch.float32 or tau.device != dev:
            raise ValueError("a per-head tau must be a float32 tensor on `device`")
        if tuple(tau.shape) == (H,):
            tau = tau.unsqueeze(0).expand(B, H)
        if tuple(tau.shape) != (B, H):
            raise ValueError("a per-head tau must have shape [B, H] or [H]")
        tau_heads = tau.contiguous()
        tau = 1.0
    filt, val = (_lib.SA_FILTER_RECALL, float(recall)) if recall is not None else \
        (_lib.SA_FILTER_LAMBDA, -math.inf if lam is None else float(lam))
    main = torch.cuda.current_stream(dev)
    h2d, d2h = _copy_streams(dev)
    with torch.cuda.device(dev):
        st = lib.sparse_attn_host(_ptr(q), _ptr(k), _ptr(v), s, float(tau), _ptr(tau_heads), filt, val, float(scale),
                                  int(bool(causal)), flags, _ptr(out), _ptr(workspace), ws_bytes, nch,
                                  ctypes.c_void_p(main.cuda_stream), ctypes.c_void_p(h2d.cuda_stream),
                                  ctypes.c_void_p(d2h.cuda_stream))
        _call("sparse_attn_host", st)
        main.synchronize()
        code = ctypes.c_int32(0)
        _call("sparse_attn_device_error", lib.sparse_attn_device_error(_stream(dev), ctypes.byref(code)))
    if code.value:
        raise SparseAttnError(f"sparse_attention (device error word {code.value})", _lib.SA_ERR_DEVICE_CHECK, lib)
    return out


def sparse_attn_device_error(device=None) -> int:
    """Read and clear the device error word (0 = no device-side check fired)."""
    lib = _lib.load()
    dev = torch.device("cuda") if device is None else torch.device(device)
    code = ctypes.c_int32(0)
    with torch.cuda.device(dev):
        _call("sparse_attn_device_error", lib.sparse_attn_device_error(_stream(dev), ctypes.byref(code)))
    return int(code.value)


def sparse_attn_selftest_wait_timeout(limit_us: int, device=None) -> None:
    """Launch the library's failure-path diagnostic on the current stream: one warp
    waits on a barrier that nothing completes, gives up after limit_us
    microseconds and records a timeout in the device error word (read it with
    sparse_attn_device_error). The kernel returns normally."""
    lib = _lib.load()
    dev = torch.device("cuda") if device is None else torch.device(device)
    with torch.cuda.device(dev):
        _call("sparse_attn_selftest_wait_timeout", lib.sparse_attn_selftest_wait_timeout(int(limit_us), _stream(dev)))
