"""Krea 2 bidirectional DiT attention core on B200 (sm_100a).

Python binding of libkrea_attn.so (C ABI in include/krea_attn.h). This module
only marshals arguments -- tensor pointers, strides, dtypes and the CUDA stream
-- and allocates outputs and workspace through torch; every step of the
attention runs in the library's CUDA kernels. There is no CPU path: calls on
tensors that are not on a CUDA device are rejected.
"""
from __future__ import annotations

import ctypes
from typing import Optional

import numpy as np
import torch

from . import _lib
from ._lib import KreaError, Params, check, lib

__all__ = ["attention", "attention_rope_q", "attention_backward", "quantize", "get_map", "map_size",
           "workspace_bytes", "workspace_layout", "bwd_scratch_bytes", "make_params", "clear_cache", "KreaError"]

_TORCH_DT = {torch.float16: "f16", torch.bfloat16: "bf16", torch.float32: "f32"}


def make_params(batch: int, q_heads: int, kv_heads: int, head_dim: int, text_len: int, grid_h: int,
                grid_w: int, *, in_dtype: str = "bf16", out_dtype: str = "f32", softmax_scale: float = 0.0,
                q_start: int = 0, q_len: int = 0, pattern: str = "band", percentage: float = 0.5,
                band_blocks: int = 2, smooth_k: bool = True, qk_fp32_accumulate: bool = False,
                window: int = 11, tile_aligned: bool = True, text_pad: int = 0,
                debug_wait_limit: int = 0, debug_flags: int = 0, overlap_previous: bool = False) -> Params:
    """krea_attn_params_t for contiguous [B, L, H, d] tensors (strides fixed up by `attention`).
    overlap_previous: the call may overlap the work before it on the stream, which must write
    nothing it reads and none of the rows it writes (e.g. the next query slice)."""
    p = Params()
    lib().krea_attn_default_params(ctypes.byref(p), batch, q_heads, kv_heads, head_dim, text_len, grid_h,
                                   grid_w)
    p.in_dtype = _lib.DTYPE[in_dtype]
    p.out_dtype = _lib.DTYPE[out_dtype]
    p.softmax_scale = float(softmax_scale)
    p.q_start = int(q_start)
    p.q_len = int(q_len)
    p.pattern = _lib.PATTERN[pattern]
    p.percentage = float(percentage)
    p.band_blocks = int(band_blocks)
    p.smooth_k = int(bool(smooth_k))
    p.qk_fp32_accumulate = int(bool(qk_fp32_accumulate))
    p.window = int(window)
    p.tile_aligned = int(bool(tile_aligned))
    p.text_pad = int(text_pad)
    p.debug_wait_limit = int(debug_wait_limit)
    p.debug_flags = int(debug_flags)
    p.overlap_previous = int(bool(overlap_previous))
    return p


def _set_strides(arr, t: torch.Tensor) -> None:
    s = t.stride()
    if t.dim() != 4 or s[3] != 1:
        raise ValueError("expected a [batch, tokens, heads, head_dim] tensor with head_dim contiguous")
    arr[0], arr[1], arr[2] = s[0], s[1], s[2]


def _stream_ptr(stream: Optional[torch.cuda.Stream], device: torch.device) -> int:
    st = stream if stream is not None else torch.cuda.current_stream(device)
    return int(st.cuda_stream)


def workspace_bytes(mode: str, text_len: int, grid_h: int, grid_w: int, params: Params) -> int:
    return int(lib().krea_attn_workspace_bytes(text_len, grid_h, grid_w, _lib.MODE[mode], ctypes.byref(params)))


def bwd_scratch_bytes(text_len: int, grid_h: int, grid_w: int, params: Params) -> int:
    """Bytes of device scratch krea_attn_bwd needs for this geometry and params."""
    return int(lib().krea_attn_bwd_scratch_bytes(text_len, grid_h, grid_w, ctypes.byref(params)))


def workspace_layout(text_len: int, grid_h: int, grid_w: int, params: Params) -> dict:
    w = _lib.WsLayout()
    check(lib().krea_attn_workspace_layout(text_len, grid_h, grid_w, _lib.MODE["tilemix"], ctypes.byref(params),
                                           ctypes.byref(w)), "workspace_layout")
    return {n: int(getattr(w, n)) for n, _ in w._fields_}


def map_size(mode: str, text_len: int, grid_h: int, grid_w: int, params: Params):
    nt, nnz = ctypes.c_int32(), ctypes.c_int32()
    check(lib().krea_attn_map_size(text_len, grid_h, grid_w, _lib.MODE[mode], ctypes.byref(params),
                                   ctypes.byref(nt), ctypes.byref(nnz)), "map_size")
    return nt.value, nnz.value


def get_map(mode: str, text_len: int, grid_h: int, grid_w: int, params: Optional[Params] = None, **opts):
    """Host copy of the tile map: (row_ptr[n_tiles+1], col[nnz], kind[nnz]) as numpy arrays."""
    if params is None:
        params = make_params(1, 1, 1, 128, text_len, grid_h, grid_w, **opts)
    nt, nnz = map_size(mode, text_len, grid_h, grid_w, params)
    row_ptr = np.zeros(nt + 1, dtype=np.int32)
    col = np.zeros(max(nnz, 1), dtype=np.int32)
    kind = np.zeros(max(nnz, 1), dtype=np.uint8)
    check(lib().krea_attn_get_map(text_len, grid_h, grid_w, _lib.MODE[mode], ctypes.byref(params),
                                  row_ptr.ctypes.data, col.ctypes.data, kind.ctypes.data, nnz), "get_map")
    return row_ptr, col[:nnz], kind[:nnz]


def get_map_device(mode: str, text_len: int, grid_h: int, grid_w: int, params: Optional[Params] = None,
                   device=None, capacity: Optional[int] = None, status: Optional[torch.Tensor] = None, **opts):
    """The tile map built on the GPU: (row_ptr[n_tiles+1] int32, col[capacity] int32,
    kind[capacity] uint8) device tensors; the first row_ptr[-1] entries are the map."""
    if params is None:
        params = make_params(1, 1, 1, 128, text_len, grid_h, grid_w, **opts)
    device = torch.device(device if device is not None else "cuda")
    nt, _ = map_size(mode, text_len, grid_h, grid_w, params)
    cap = nt * nt if capacity is None else capacity
    row_ptr = torch.empty(nt + 1, dtype=torch.int32, device=device)
    col = torch.empty(max(cap, 1), dtype=torch.int32, device=device)
    kind = torch.empty(max(cap, 1), dtype=torch.uint8, device=device)
    if status is not None:
        params.status = status.data_ptr()
    stream = torch.cuda.current_stream(device).cuda_stream
    check(lib().krea_attn_build_map_device(text_len, grid_h, grid_w, _lib.MODE[mode], ctypes.byref(params),
                                           row_ptr.data_ptr(), col.data_ptr(), kind.data_ptr(), cap, stream),
          "build_map_device")
    return row_ptr, col, kind


def rope_positions(text_len: int, grid_h: int, grid_w: int, device=None) -> torch.Tensor:
    """[L, 3] int32 rotary positions of the joint sequence, from krea_attn_rope_positions
    (host work in the library), moved to `device` when given."""
    L = text_len + grid_h * grid_w
    pos = torch.zeros(max(L, 1), 3, dtype=torch.int32)
    check(lib().krea_attn_rope_positions(text_len, grid_h, grid_w, pos.data_ptr(), pos.shape[0]),
          "rope_positions")
    return pos.to(device) if device is not None else pos


def rope_params(head_dim: int = 128, axes_dim=None, theta: Optional[float] = None,
                eps: Optional[float] = None) -> _lib.RopeParams:
    r = _lib.RopeParams()
    lib().krea_attn_default_rope(ctypes.byref(r), head_dim)
    if axes_dim is not None:
        for i in range(3):
            r.axes_dim[i] = int(axes_dim[i])
    if theta is not None:
        r.theta = float(theta)
    if eps is not None:
        r.eps = float(eps)
    return r


def rope_table(pos: torch.Tensor, rope: Optional[_lib.RopeParams] = None, head_dim: int = 128,
               stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    """(cos, sin) table [L, n_pairs, 2] fp32 on pos's device, for krea_attn_qk_prologue."""
    _check_inputs(pos)
    rope = rope if rope is not None else rope_params(head_dim)
    pos = pos.to(torch.int32).contiguous()
    n_pairs = sum(rope.axes_dim) // 2
    table = torch.empty(pos.shape[0], n_pairs, 2, dtype=torch.float32, device=pos.device)
    check(lib().krea_attn_rope_table(pos.data_ptr(), pos.shape[0], ctypes.byref(rope), table.data_ptr(),
                                     _stream_ptr(stream, pos.device)), "rope_table")
    return table


def qk_prologue(x: torch.Tensor, table: torch.Tensor, gamma: Optional[torch.Tensor] = None,
                out: Optional[torch.Tensor] = None, rope: Optional[_lib.RopeParams] = None,
                with_codes: bool = False, stream: Optional[torch.cuda.Stream] = None):
    """rope(rmsnorm(x)) for x [B, L, H, d] fp16/bf16 (out may be x). With with_codes,
    also returns the INT8 codes [B, L, H, d] and block scales [B, H, ceil(L/128)]."""
    _check_inputs(x, table, gamma, out)
    B, L, H, d = x.shape
    rope = rope if rope is not None else rope_params(d)
    y = out if out is not None else torch.empty_like(x)
    codes = scales = None
    if with_codes:
        codes = torch.empty(B, L, H, d, dtype=torch.int8, device=x.device)
        scales = torch.empty(B, H, -(-L // 128), dtype=torch.float32, device=x.device)
    dt = {torch.float16: _lib.DTYPE["f16"], torch.bfloat16: _lib.DTYPE["bf16"]}.get(x.dtype, _lib.DTYPE["f32"])
    xs = (ctypes.c_int64 * 3)(*x.stride()[:3])
    ys = (ctypes.c_int64 * 3)(*y.stride()[:3])
    g = gamma.to(torch.float32).contiguous() if gamma is not None else None
    check(lib().krea_attn_qk_prologue(x.data_ptr(), y.data_ptr(), g.data_ptr() if g is not None else None,
                                      table.data_ptr(), B, L, H, d, dt, xs, ys, ctypes.byref(rope),
                                      codes.data_ptr() if codes is not None else None,
                                      scales.data_ptr() if scales is not None else None,
                                      _stream_ptr(stream, x.device)), "qk_prologue")
    return (y, codes, scales) if with_codes else y


def _check_inputs(*ts):
    for t in ts:
        if t is not None and not t.is_cuda:
            raise ValueError("krea attention runs on CUDA tensors only")


def _forward_params(q, k, v, gate, out, out_dtype, workspace, status, lse, mode, text_len, grid_h, grid_w, opts):
    """The output tensor and krea_attn_params_t of a forward call (argument marshalling)."""
    B, L, Hq, d = q.shape
    Hkv = k.shape[2]
    in_dt = _TORCH_DT[q.dtype]
    if out is None:
        odt = out_dtype if out_dtype is not None else q.dtype
        out = torch.empty((B, L, Hq, d), dtype=odt, device=q.device)
    p = make_params(B, Hq, Hkv, d, text_len, grid_h, grid_w, in_dtype=in_dt, out_dtype=_TORCH_DT[out.dtype],
                    **opts)
    _set_strides(p.q_stride, q)
    _set_strides(p.k_stride, k)
    _set_strides(p.v_stride, v)
    _set_strides(p.out_stride, out)
    if gate is not None:
        _set_strides(p.gate_stride, gate)
    if mode == "tilemix":
        need = workspace_bytes(mode, text_len, grid_h, grid_w, p)
        if workspace is None:
            workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
        p.workspace = workspace.data_ptr()
        p.workspace_bytes = workspace.numel() * workspace.element_size()
    if lse is not None:  # [B, Hq, L] fp32: ln sum_j exp(scale s_ij) per valid query row
        if lse.dtype != torch.float32 or not lse.is_contiguous() or tuple(lse.shape) != (B, Hq, L):
            raise ValueError("lse must be a contiguous float32 tensor of shape [B, Hq, L]")
        p.lse = lse.data_ptr()
    if status is not None:
        p.status = status.data_ptr()
    return out, p


def attention(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, gate: Optional[torch.Tensor] = None, *,
              text_len: int, grid_h: int, grid_w: int, mode: str = "dense",
              out: Optional[torch.Tensor] = None, out_dtype: Optional[torch.dtype] = torch.float32,
              workspace: Optional[torch.Tensor] = None, status: Optional[torch.Tensor] = None,
              stream: Optional[torch.cuda.Stream] = None, lse: Optional[torch.Tensor] = None,
              **opts) -> torch.Tensor:
    """out = sigmoid(gate) * softmax(scale q k^T over the admitted keys) v, per query head.

    q [B, L, Hq, d], k and v [B, L, Hkv, d], gate [B, L, Hq, d] or None; L = text_len + grid_h * grid_w.
    mode: "dense" | "tilemix" | "scanline"; `opts` are make_params keywords (q_start, q_len,
    pattern, percentage, band_blocks, smooth_k, window, tile_aligned, text_pad, ...).
    """
    _check_inputs(q, k, v, gate, out, workspace, status, lse)
    out, p = _forward_params(q, k, v, gate, out, out_dtype, workspace, status, lse, mode, text_len, grid_h,
                             grid_w, opts)
    rc = lib().krea_attn_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(),
                             gate.data_ptr() if gate is not None else None, out.data_ptr(),
                             text_len, grid_h, grid_w, _lib.MODE[mode], ctypes.byref(p),
                             _stream_ptr(stream, q.device))
    check(rc, "krea_attn_fwd")
    return out


def attention_rope_q(q_raw: torch.Tensor, k: torch.Tensor, v: torch.Tensor, gate: Optional[torch.Tensor],
                     table: torch.Tensor, q_gamma: Optional[torch.Tensor] = None,
                     rope: Optional[_lib.RopeParams] = None, *, text_len: int, grid_h: int, grid_w: int,
                     mode: str = "dense", out: Optional[torch.Tensor] = None,
                     out_dtype: Optional[torch.dtype] = torch.float32, status: Optional[torch.Tensor] = None,
                     stream: Optional[torch.cuda.Stream] = None, lse: Optional[torch.Tensor] = None,
                     **opts) -> torch.Tensor:
    """attention(qk_prologue(q_raw, table, q_gamma), k, v, gate) in one kernel: the
    query prologue runs on each Q tile in shared memory (krea_attn_fwd_rope_q).
    k must already be through qk_prologue; table from rope_table with `rope`.
    Dense and scanline modes."""
    _check_inputs(q_raw, k, v, gate, table, q_gamma, out, status, lse)
    d = q_raw.shape[3]
    rope = rope if rope is not None else rope_params(d)
    g = q_gamma.to(torch.float32).contiguous() if q_gamma is not None else None
    out, p = _forward_params(q_raw, k, v, gate, out, out_dtype, None, status, lse, mode, text_len, grid_h,
                             grid_w, opts)
    rc = lib().krea_attn_fwd_rope_q(q_raw.data_ptr(), g.data_ptr() if g is not None else None, table.data_ptr(),
                                    ctypes.byref(rope), k.data_ptr(), v.data_ptr(),
                                    gate.data_ptr() if gate is not None else None, out.data_ptr(),
                                    text_len, grid_h, grid_w, _lib.MODE[mode], ctypes.byref(p),
                                    _stream_ptr(stream, q_raw.device))
    check(rc, "krea_attn_fwd_rope_q")
    return out


def attention_backward(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, gate: Optional[torch.Tensor],
                       out: torch.Tensor, dout: torch.Tensor, lse: torch.Tensor, *, text_len: int, grid_h: int,
                       grid_w: int, mode: str = "dense", stream: Optional[torch.cuda.Stream] = None,
                       status: Optional[torch.Tensor] = None, scratch: Optional[torch.Tensor] = None,
                       grads: Optional[tuple] = None, **opts):
    """(dq, dk, dv, dgate) of krea_attn_fwd's output (fp32 tensors; dgate None without
    a gate). out, dout: the forward's output and its gradient, contiguous, same dtype;
    lse: the forward's [B, Hq, L] log-sum-exp (attention(..., lse=...)).
    scratch (krea_attn_bwd_scratch_bytes bytes, uint8) and grads (dq, dk, dv, dgate:
    contiguous fp32 tensors) may be passed in to reuse memory across calls."""
    _check_inputs(q, k, v, gate, out, dout, lse, status)
    B, L, Hq, d = q.shape
    Hkv = k.shape[2]
    in_dt = _TORCH_DT[q.dtype]
    p = make_params(B, Hq, Hkv, d, text_len, grid_h, grid_w, in_dtype=in_dt, out_dtype=_TORCH_DT[out.dtype],
                    **opts)
    for arr, t in ((p.q_stride, q), (p.k_stride, k), (p.v_stride, v)):
        arr[0], arr[1], arr[2] = t.stride()[:3]
    if gate is not None:
        p.gate_stride[0], p.gate_stride[1], p.gate_stride[2] = gate.stride()[:3]
    if status is not None:
        p.status = status.data_ptr()
    out, dout = out.contiguous(), dout.contiguous()
    if grads is not None:
        dq, dk, dv, dgate = grads
        _check_inputs(dq, dk, dv, dgate)
        for t, shape in ((dq, (B, L, Hq, d)), (dk, (B, L, Hkv, d)), (dv, (B, L, Hkv, d)), (dgate, (B, L, Hq, d))):
            if t is not None and (t.dtype != torch.float32 or not t.is_contiguous() or tuple(t.shape) != shape):
                raise ValueError("grads must be contiguous float32 tensors of the gradient shapes")
        if gate is None:
            dgate = None
    else:
        dq = torch.empty(B, L, Hq, d, dtype=torch.float32, device=q.device)
        dk = torch.empty(B, L, Hkv, d, dtype=torch.float32, device=q.device)
        dv = torch.empty(B, L, Hkv, d, dtype=torch.float32, device=q.device)
        dgate = torch.empty(B, L, Hq, d, dtype=torch.float32, device=q.device) if gate is not None else None
    need = bwd_scratch_bytes(text_len, grid_h, grid_w, p)
    if scratch is None:
        scratch = torch.empty(need, dtype=torch.uint8, device=q.device)
    else:
        _check_inputs(scratch)
        if scratch.numel() * scratch.element_size() < need:
            raise ValueError(f"scratch holds {scratch.numel() * scratch.element_size()} bytes, {need} needed")
    check(lib().krea_attn_bwd(q.data_ptr(), k.data_ptr(), v.data_ptr(),
                              gate.data_ptr() if gate is not None else None, out.data_ptr(), dout.data_ptr(),
                              lse.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(),
                              dgate.data_ptr() if dgate is not None else None, scratch.data_ptr(),
                              text_len, grid_h, grid_w, _lib.MODE[mode], ctypes.byref(p),
                              _stream_ptr(stream, q.device)), "krea_attn_bwd")
    return dq, dk, dv, dgate


def quantize(q: torch.Tensor, k: torch.Tensor, *, text_len: int, grid_h: int, grid_w: int,
             smooth_k: bool = True, workspace: Optional[torch.Tensor] = None,
             stream: Optional[torch.cuda.Stream] = None) -> dict:
    """Run only the TileMix quantiser; returns views of the workspace:
    kc (centred keys), q8, k8, sq, sk, mu."""
    _check_inputs(q, k, workspace)
    B, L, Hq, d = q.shape
    Hkv = k.shape[2]
    p = make_params(B, Hq, Hkv, d, text_len, grid_h, grid_w, in_dtype=_TORCH_DT[q.dtype], smooth_k=smooth_k)
    _set_strides(p.q_stride, q)
    _set_strides(p.k_stride, k)
    lay = workspace_layout(text_len, grid_h, grid_w, p)
    if workspace is None:
        workspace = torch.empty(lay["total"], dtype=torch.uint8, device=q.device)
    p.workspace = workspace.data_ptr()
    p.workspace_bytes = workspace.numel()
    check(lib().krea_attn_quantize(q.data_ptr(), k.data_ptr(), text_len, grid_h, grid_w, ctypes.byref(p),
                                   _stream_ptr(stream, q.device)), "krea_attn_quantize")
    nt = (L + _lib.TILE - 1) // _lib.TILE

    def view(off, n, dt, shape):
        return workspace[off:off + n * torch.tensor([], dtype=dt).element_size()].view(dt).view(shape)

    res = {
        "q8": view(lay["q8"], B * L * Hq * d, torch.int8, (B, L, Hq, d)),
        "k8": view(lay["k8"], B * L * Hkv * d, torch.int8, (B, L, Hkv, d)),
        "sq": view(lay["sq"], B * Hq * nt, torch.float32, (B, Hq, nt)),
        "sk": view(lay["sk"], B * Hkv * nt, torch.float32, (B, Hkv, nt)),
        "workspace": workspace,
    }
    if smooth_k:
        res["kc"] = view(lay["kc"], B * L * Hkv * d, q.dtype, (B, L, Hkv, d))
        res["mu"] = view(lay["mu"], B * Hkv * d, torch.float32, (B, Hkv, d))
    return res


def clear_cache() -> None:
    lib().krea_attn_clear_cache()
