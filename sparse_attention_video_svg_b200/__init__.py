"""B200 (sm_100a) sparse spatial/temporal 3D attention for video DiTs.

Thin Python binding of the C ABI in include/svg.h (libsvg_b200.so).  Each
function below marshals torch tensors into pointers, sizes and the current
CUDA stream and calls the entry point of the same name; every step of the
computation runs in the library's CUDA kernels.  torch is used only to
allocate device memory (outputs and scratch the caller did not pass) and to
name the stream.

The layer the library implements (Sparse VideoGen article,
m.jxzklqfsx.com/article/815093.html; CalibAtt article, lpnh.cn/news/568491):

    mse, mode = svg_profile_heads(q, k, v, F, P, w, sample_idx)
    lists     = geometric_lists(F, P, w, N)            # spatial, temporal, dense
    q', k', v' = svg_permute_token_major(x, F, P, mode)  for x in (q, k, v)
    o'        = svg_sparse_attn(q', k', v', mode, *lists)
    o         = svg_permute_frame_major(o', F, P, mode)

``svg_layer`` runs exactly that sequence (optionally after
``svg_qk_norm_rope``, QK-Norm + RoPE of q and k).
"""
from __future__ import annotations

from typing import NamedTuple, Optional, Sequence

import ctypes as C

import torch

from . import _lib
from ._lib import (SVG_BF16, SVG_FP32, SVG_MODE_DENSE, SVG_MODE_SPATIAL, SVG_MODE_TEMPORAL,
                   SVG_TILE, SvgError)

__all__ = [
    "SVG_MODE_SPATIAL", "SVG_MODE_TEMPORAL", "SVG_MODE_DENSE", "SVG_TILE", "SvgError",
    "BlockLists", "svg_version", "svg_profile_heads", "svg_profile_heads_noalloc",
    "svg_permute_token_major", "svg_permute_temporal_heads",
    "svg_permute_frame_major", "svg_build_block_mask", "svg_block_energy",
    "svg_build_block_mask_calibrated", "svg_sparse_attn", "svg_sparse_attn_fused",
    "svg_v_exponents", "svg_pair_query_tiles", "svg_layer_from_host", "HostLayerBuffers",
    "svg_attention_from_host",
    "svg_epsilon_schedule", "svg_lists_to_intervals", "svg_lists_to_bitmap", "geometric_lists",
    "QKTransform", "svg_qk_norm_rope", "svg_row_similarity", "svg_anchor_lists",
    "svg_anchor_list_ids", "svg_row_broadcast", "svg_repeat_attention", "svg_layer",
    "n_tiles",
]


def n_tiles(N: int) -> int:
    return (N + SVG_TILE - 1) // SVG_TILE


def svg_version() -> str:
    return _lib.lib.svg_version().decode()


def _dt(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return SVG_BF16
    if t.dtype == torch.float32:
        return SVG_FP32
    raise TypeError(f"unsupported dtype {t.dtype} (bf16 or float32)")


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _check_qkv(*ts: torch.Tensor):
    t0 = ts[0]
    for t in ts:
        if t.dim() != 4 or not t.is_cuda or not t.is_contiguous():
            raise ValueError("tensors must be contiguous CUDA [B, H, N, d]")
        if t.shape != t0.shape or t.dtype != t0.dtype:
            raise ValueError("q, k, v must share shape and dtype")
    return t0.shape


def _scratch(nbytes: int, device) -> torch.Tensor:
    # torch's caching allocator hands out 512-byte aligned blocks
    return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)


class BlockLists(NamedTuple):
    """Several CSR key-block lists sharing one indices buffer.
    indptr: int32 [n_lists * (n_qblocks + 1)], absolute offsets into indices."""
    indptr: torch.Tensor
    indices: torch.Tensor
    n_lists: int
    n_qblocks: int
    # optional int32 [n_lists * n_qblocks]: per list, the order in which the
    # attention kernel pairs query tiles (scheduling only)
    tile_order: Optional[torch.Tensor] = None


# --------------------------------------------------------------------- steps

def svg_profile_heads(q, k, v, frames: int, tokens_per_frame: int, spatial_width: int,
                      sample_idx: torch.Tensor, *, mse_out=None, mode_out=None, workspace=None,
                      stream=None):
    """Online profiling; returns (mse [B*H, 2] float32, mode [B*H] int32)."""
    B, H, N, d = _check_qkv(q, k, v)
    S = sample_idx.numel()
    dev = q.device
    if mse_out is None:
        mse_out = torch.empty(B * H, 2, dtype=torch.float32, device=dev)
    if mode_out is None:
        mode_out = torch.empty(B * H, dtype=torch.int32, device=dev)
    need = _lib.lib.svg_profile_workspace_size(B, H, N, d, S)
    if workspace is None:
        workspace = _scratch(need, dev)
    _lib.call("svg_profile_heads", q.data_ptr(), k.data_ptr(), v.data_ptr(), _dt(q), B, H, N, d,
              frames, tokens_per_frame, spatial_width, sample_idx.data_ptr(), S,
              mse_out.data_ptr(), mode_out.data_ptr(), workspace.data_ptr(), workspace.numel(),
              _stream(stream))
    return mse_out, mode_out


def svg_profile_heads_noalloc(q, k, v, frames: int, tokens_per_frame: int, spatial_width: int,
                              sample_idx: torch.Tensor, *, mse_out=None, mode_out=None,
                              stream=None):
    """svg_profile_heads with the library's fixed device scratch instead of a
    workspace (for callers that cannot allocate); returns (mse, mode)."""
    B, H, N, d = _check_qkv(q, k, v)
    dev = q.device
    if mse_out is None:
        mse_out = torch.empty(B * H, 2, dtype=torch.float32, device=dev)
    if mode_out is None:
        mode_out = torch.empty(B * H, dtype=torch.int32, device=dev)
    _lib.call("svg_profile_heads_noalloc", q.data_ptr(), k.data_ptr(), v.data_ptr(), _dt(q), B,
              H, N, d, frames, tokens_per_frame, spatial_width, sample_idx.data_ptr(),
              sample_idx.numel(), mse_out.data_ptr(), mode_out.data_ptr(), _stream(stream))
    return mse_out, mode_out


def _permute(name, x, frames, tokens_per_frame, mode, out, stream):
    B, H, N, d = _check_qkv(x)
    if out is None:
        out = torch.empty_like(x)
    _lib.call(name, x.data_ptr(), out.data_ptr(), _dt(x), B, H, N, d, frames, tokens_per_frame,
              _ptr(mode), _stream(stream))
    return out


def svg_permute_token_major(x, frames: int, tokens_per_frame: int, mode=None, out=None,
                            stream=None):
    """y[b,h,s*F+f] = x[b,h,f*P+s] for TEMPORAL heads (all heads if mode is None)."""
    return _permute("svg_permute_token_major", x, frames, tokens_per_frame, mode, out, stream)


def svg_permute_temporal_heads(x, frames: int, tokens_per_frame: int, mode, out=None,
                               stream=None):
    """svg_permute_token_major for TEMPORAL heads only; the other heads of
    `out` are not written (the copy the fused attention reads)."""
    if mode is None:
        raise ValueError("svg_permute_temporal_heads needs the modes")
    return _permute("svg_permute_temporal_heads", x, frames, tokens_per_frame, mode, out, stream)


def svg_permute_frame_major(x, frames: int, tokens_per_frame: int, mode=None, out=None,
                            stream=None):
    """The inverse of svg_permute_token_major."""
    return _permute("svg_permute_frame_major", x, frames, tokens_per_frame, mode, out, stream)


def svg_build_block_mask(kind: int, frames: int, tokens_per_frame: int, spatial_width: int,
                         N: int, *, indptr=None, indices=None, index_base: int = 0, nnz=None,
                         status=None, device=None, stream=None):
    """Geometric key-block list of one kind; returns (indptr, indices, nnz).
    indices has capacity nB*nB unless given; nnz is a device int64 [1]."""
    nb = n_tiles(N)
    device = device or torch.device("cuda")
    if indptr is None:
        indptr = torch.empty(nb + 1, dtype=torch.int32, device=device)
    if indices is None:
        indices = torch.empty(nb * nb, dtype=torch.int32, device=device)
    if nnz is None:
        nnz = torch.empty(1, dtype=torch.int64, device=device)
    _lib.call("svg_build_block_mask", kind, frames, tokens_per_frame, spatial_width, N,
              indptr.data_ptr(), indices.data_ptr(), indices.numel(), index_base, nnz.data_ptr(),
              _ptr(status), _stream(stream))
    return indptr, indices, nnz


def geometric_lists(frames: int, tokens_per_frame: int, spatial_width: int, N: int,
                    device=None, stream=None) -> BlockLists:
    """The spatial, temporal and dense lists in one BlockLists (list id = mode)."""
    nb = n_tiles(N)
    device = device or torch.device("cuda")
    indptr = torch.empty(3 * (nb + 1), dtype=torch.int32, device=device)
    indices = torch.empty(3 * nb * nb, dtype=torch.int32, device=device)
    for kind in (SVG_MODE_SPATIAL, SVG_MODE_TEMPORAL, SVG_MODE_DENSE):
        base = kind * nb * nb
        svg_build_block_mask(kind, frames, tokens_per_frame, spatial_width, N,
                             indptr=indptr[kind * (nb + 1):(kind + 1) * (nb + 1)],
                             indices=indices[base:base + nb * nb], index_base=base,
                             device=device, stream=stream)
    return BlockLists(indptr, indices, 3, nb)


def svg_block_energy(q, k, *, out=None, workspace=None, stream=None):
    """Dense block energy E [B*H, nB, nB] (float32)."""
    B, H, N, d = _check_qkv(q, k)
    nb = n_tiles(N)
    if out is None:
        out = torch.empty(B * H, nb, nb, dtype=torch.float32, device=q.device)
    if workspace is None:
        workspace = _scratch(_lib.lib.svg_block_energy_workspace_size(B, H, N), q.device)
    _lib.call("svg_block_energy", q.data_ptr(), k.data_ptr(), _dt(q), B, H, N, d, out.data_ptr(),
              workspace.data_ptr(), workspace.numel(), _stream(stream))
    return out


def svg_build_block_mask_calibrated(energy: torch.Tensor, eps: float, rho: float, *,
                                    status=None, stream=None) -> BlockLists:
    """energy [R, L, nQB, nKB] float32 -> one list per L (BlockLists)."""
    if energy.dim() != 4 or energy.dtype != torch.float32 or not energy.is_contiguous():
        raise ValueError("energy must be contiguous float32 [R, L, nQB, nKB]")
    R, L, nq, nk = energy.shape
    dev = energy.device
    indptr = torch.empty(L * (nq + 1), dtype=torch.int32, device=dev)
    indices = torch.empty(L * nq * nk, dtype=torch.int32, device=dev)
    nnz = torch.empty(1, dtype=torch.int64, device=dev)
    ws = _scratch(_lib.lib.svg_calibrated_workspace_size(L, nq, nk), dev)
    _lib.call("svg_build_block_mask_calibrated", energy.data_ptr(), R, L, nq, nk, float(eps),
              float(rho), indptr.data_ptr(), indices.data_ptr(), indices.numel(), nnz.data_ptr(),
              _ptr(status), ws.data_ptr(), ws.numel(), _stream(stream))
    return BlockLists(indptr, indices, L, nq)


def svg_sparse_attn(q, k, v, list_id: torch.Tensor, lists: BlockLists, *, scale: float = 0.0,
                    v_exp=None, out=None, status=None, stream=None):
    """Block-sparse attention over 128x128 tiles; returns o [B, H, N, d].
    v_exp: optional int32 [B*H] from svg_v_exponents (V scaled into the fp16
    range of the P.V product)."""
    B, H, N, d = _check_qkv(q, k, v)
    if out is None:
        out = torch.empty_like(q)
    _lib.call("svg_sparse_attn", q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), _dt(q),
              B, H, N, d, list_id.data_ptr(), lists.n_lists, lists.n_qblocks,
              lists.indptr.data_ptr(), lists.indices.data_ptr(), float(scale), _ptr(status),
              _ptr(v_exp), _stream(stream))
    return out


def svg_v_exponents(v, *, out=None, stream=None):
    """Per-head exponents e (int32 [B*H]) with max|v| * 2^-e <= 65504."""
    B, H, N, d = _check_qkv(v)
    if out is None:
        out = torch.empty(B * H, dtype=torch.int32, device=v.device)
    _lib.call("svg_v_exponents", v.data_ptr(), _dt(v), B, H, N, d, out.data_ptr(), _stream(stream))
    return out


def svg_sparse_attn_fused(q, k, v, frames: int, tokens_per_frame: int, mode: torch.Tensor,
                          lists: BlockLists, *, layout: int = 3, copies=None, scale: float = 0.0,
                          v_exp=None, out=None, status=None, stream=None):
    """Block-sparse attention with the token-major reordering of temporal
    heads fused in: layout bit 1 (SVG_FUSE_INPUT) gathers q, k, v from
    frame-major memory, bit 2 (SVG_FUSE_OUTPUT) writes o frame-major.
    copies = (q_tm, k_tm, v_tm): token-major copies of every head, read by
    the temporal heads instead (q, k, v then frame-major)."""
    B, H, N, d = _check_qkv(q, k, v)
    if out is None:
        out = torch.empty_like(q)
    qt, kt, vt = (None, None, None) if copies is None else (c.data_ptr() for c in copies)
    _lib.call("svg_sparse_attn_fused", q.data_ptr(), k.data_ptr(), v.data_ptr(), qt, kt, vt,
              out.data_ptr(), _dt(q), B, H, N, d, frames, tokens_per_frame, mode.data_ptr(),
              int(layout), lists.n_lists, lists.n_qblocks, lists.indptr.data_ptr(),
              lists.indices.data_ptr(), _ptr(lists.tile_order), float(scale), _ptr(status),
              _ptr(v_exp), _stream(stream))
    return out


def svg_pair_query_tiles(lists: BlockLists, n_kblocks: Optional[int] = None, *, status=None,
                         stream=None) -> BlockLists:
    """The lists with a pairing order of their query tiles (tile_order): per
    list, consecutive pairs share many key blocks (greedy, on the GPU).  For
    lists built once and used for many steps; the attention results do not
    depend on it.  n_kblocks defaults to n_qblocks (square lists)."""
    nk = lists.n_qblocks if n_kblocks is None else int(n_kblocks)
    dev = lists.indptr.device
    ws = _scratch(_lib.lib.svg_pair_query_tiles_workspace_size(lists.n_lists, lists.n_qblocks, nk),
                  dev)
    order = torch.empty(lists.n_lists * lists.n_qblocks, dtype=torch.int32, device=dev)
    _lib.call("svg_pair_query_tiles", lists.indptr.data_ptr(), lists.indices.data_ptr(),
              lists.n_lists, lists.n_qblocks, nk, order.data_ptr(), _ptr(status), ws.data_ptr(),
              ws.numel(), _stream(stream))
    return lists._replace(tile_order=order)


class QKTransform(NamedTuple):
    """Parameters of the QK-Norm + RoPE step before attention: per-channel
    weights (float32 [d] CUDA tensors, or None for 1), epsilon, and the rotary
    tables cos, sin (float32 [N, d/2] CUDA tensors, or None for no RoPE)."""
    gamma_q: Optional[torch.Tensor]
    gamma_k: Optional[torch.Tensor]
    eps: float
    cos: Optional[torch.Tensor]
    sin: Optional[torch.Tensor]
    norm: bool = True


def svg_qk_norm_rope(q, k, qk: QKTransform, *, out=None, tm_out=None, frames: int = 0,
                     tokens_per_frame: int = 0, stream=None):
    """QK-Norm then RoPE of q and k in one pass.  out = (q_out, k_out)
    (allocated when None; may be (q, k) for in place); tm_out = (q_tm, k_tm)
    also writes the token-major copies of every head (needs frames and
    tokens_per_frame).  Returns (q_out, k_out)."""
    B, H, N, d = _check_qkv(q, k)
    if out is None:
        out = (torch.empty_like(q), torch.empty_like(k))
    _check_qkv(q, *out)
    qt, kt = (None, None) if tm_out is None else (tm_out[0].data_ptr(), tm_out[1].data_ptr())
    if tm_out is not None:
        _check_qkv(q, *tm_out)
    ops = (_lib.SVG_QK_NORM if qk.norm else 0) | (_lib.SVG_QK_ROPE if qk.cos is not None else 0)
    for t in (qk.gamma_q, qk.gamma_k, qk.cos, qk.sin):
        if t is not None and (t.dtype != torch.float32 or not t.is_cuda or not t.is_contiguous()):
            raise ValueError("QK-Norm weights and RoPE tables must be contiguous float32 CUDA")
    _lib.call("svg_qk_norm_rope", q.data_ptr(), k.data_ptr(), out[0].data_ptr(),
              out[1].data_ptr(), qt, kt, _dt(q), B, H, N, d, int(frames), int(tokens_per_frame),
              ops, _ptr(qk.gamma_q), _ptr(qk.gamma_k), float(qk.eps), _ptr(qk.cos), _ptr(qk.sin),
              _stream(stream))
    return out


# ------------------------------------------------ spatial-repetition heads

def svg_row_similarity(q, k, frames: int, rows: int, cols: int, eval_frames=None, *,
                       n_frames: Optional[int] = None, out=None, workspace=None, status=None,
                       stream=None):
    """Mean row-pattern cosine similarity per head ([CAL] 3.2) over the
    frames in eval_frames (int32 CUDA tensor) or frames 0 .. n_frames-1
    (all frames when both are None).  Returns float32 [B*H]."""
    B, H, N, d = _check_qkv(q, k)
    if eval_frames is None:
        nf = frames if n_frames is None else int(n_frames)
        fptr = None
    else:
        nf = eval_frames.numel()
        fptr = eval_frames.data_ptr()
    if out is None:
        out = torch.empty(B * H, dtype=torch.float32, device=q.device)
    if workspace is None:
        workspace = _scratch(_lib.lib.svg_row_similarity_workspace_size(
            _dt(q), B, H, rows, cols, nf), q.device)
    _lib.call("svg_row_similarity", q.data_ptr(), k.data_ptr(), _dt(q), B, H, N, d, frames, rows,
              cols, fptr, nf, out.data_ptr(), workspace.data_ptr(), workspace.numel(),
              _ptr(status), _stream(stream))
    return out


def svg_anchor_lists(lists: BlockLists, N: int, frames: int, rows: int, cols: int,
                     list_id: Optional[torch.Tensor] = None,
                     repeat: Optional[torch.Tensor] = None, *, anchors: int = 5,
                     skip_list: int = -1, status=None, stream=None):
    """Lists 0 .. L-1 unchanged, L .. 2L-1 with anchor-free query tiles
    emptied (with a pairing order that puts the tiles with work first);
    repeating heads move to the second half.  Returns (BlockLists with 2L
    lists, list_id_out), list_id_out None when list_id is None."""
    L, nqb = lists.n_lists, lists.n_qblocks
    dev = lists.indptr.device
    indptr = torch.empty(2 * L * (nqb + 1), dtype=torch.int32, device=dev)
    cap = max(2 * lists.indices.numel(), 1)
    indices = torch.empty(cap, dtype=torch.int32, device=dev)
    ids = None if list_id is None else torch.empty_like(list_id)
    order = torch.empty(2 * L * nqb, dtype=torch.int32, device=dev)
    _lib.call("svg_anchor_lists", L, nqb, lists.indptr.data_ptr(), lists.indices.data_ptr(), N,
              frames, rows, cols, int(anchors), _ptr(list_id), _ptr(repeat),
              0 if list_id is None else list_id.numel(), int(skip_list), indptr.data_ptr(),
              indices.data_ptr(), cap, _ptr(ids), order.data_ptr(), _ptr(status),
              _stream(stream))
    return BlockLists(indptr, indices, 2 * L, nqb, order), ids


def svg_anchor_list_ids(list_id: torch.Tensor, repeat: Optional[torch.Tensor], n_lists: int, *,
                        skip_list: int = -1, out=None, stream=None):
    """list_id + n_lists for heads with repeat != 0 (and a list other than
    skip_list), list_id otherwise."""
    if out is None:
        out = torch.empty_like(list_id)
    _lib.call("svg_anchor_list_ids", list_id.data_ptr(), _ptr(repeat), list_id.numel(),
              int(n_lists), int(skip_list), out.data_ptr(), _stream(stream))
    return out


def svg_row_broadcast(o, frames: int, rows: int, cols: int, list_id: torch.Tensor, n_lists: int,
                      *, anchors: int = 5, stream=None):
    """In place: non-anchor rows of heads with list_id >= n_lists take their
    anchor row's output."""
    B, H, N, d = _check_qkv(o)
    _lib.call("svg_row_broadcast", o.data_ptr(), _dt(o), B, H, N, d, frames, rows, cols,
              int(anchors), list_id.data_ptr(), int(n_lists), _stream(stream))
    return o


def svg_repeat_attention(q, k, v, frames: int, rows: int, cols: int, list_id: torch.Tensor,
                         lists: BlockLists, repeat: torch.Tensor, *, anchors: int = 5,
                         skip_list: int = -1, out=None, status=None, stream=None):
    """Block-sparse attention in which heads flagged in `repeat` compute
    only the query tiles holding anchor rows and broadcast the anchors'
    outputs to the other rows."""
    N = q.shape[2]
    alists, ids = svg_anchor_lists(lists, N, frames, rows, cols, list_id, repeat,
                                   anchors=anchors, skip_list=skip_list, status=status,
                                   stream=stream)
    # layout 0: svg_sparse_attn with list_id = ids, plus the pairing order
    o = svg_sparse_attn_fused(q, k, v, frames, rows * cols, ids, alists, layout=0, out=out,
                              status=status, stream=stream)
    svg_row_broadcast(o, frames, rows, cols, ids, lists.n_lists, anchors=anchors, stream=stream)
    return o


# ------------------------------------------- threshold schedule, mask encodings

def svg_epsilon_schedule(n_steps: int, eps_first: float = 0.99, eps_last: float = 0.84):
    """Energy threshold for each denoising step (host computation)."""
    out = (C.c_double * max(n_steps, 1))()
    _lib.call("svg_epsilon_schedule", int(n_steps), float(eps_first), float(eps_last),
              C.cast(out, C.c_void_p))
    return [out[i] for i in range(n_steps)]


def svg_lists_to_intervals(indptr: torch.Tensor, indices: torch.Tensor, n_cols: int, *,
                           status=None, stream=None):
    """CSR rows -> skip list of maximal block runs: (iptr, starts, ends)."""
    n_rows = indptr.numel() - 1
    dev = indptr.device
    iptr = torch.empty(n_rows + 1, dtype=torch.int32, device=dev)
    n = torch.zeros(1, dtype=torch.int64, device=dev)
    _lib.call("svg_lists_to_intervals", n_rows, int(n_cols), indptr.data_ptr(),
              indices.data_ptr(), iptr.data_ptr(), None, None, 0, n.data_ptr(), _ptr(status),
              _stream(stream))
    cap = max(int(n.item()), 1)
    starts = torch.empty(cap, dtype=torch.int32, device=dev)
    ends = torch.empty(cap, dtype=torch.int32, device=dev)
    _lib.call("svg_lists_to_intervals", n_rows, int(n_cols), indptr.data_ptr(),
              indices.data_ptr(), iptr.data_ptr(), starts.data_ptr(), ends.data_ptr(), cap,
              n.data_ptr(), _ptr(status), _stream(stream))
    total = int(n.item())
    return iptr, starts[:total], ends[:total]


def svg_lists_to_bitmap(indptr: torch.Tensor, indices: torch.Tensor, n_cols: int, *,
                        out=None, status=None, stream=None):
    """CSR rows -> bitmap, uint32 words [rows][ceil(n_cols / 32)] (as int32)."""
    n_rows = indptr.numel() - 1
    if out is None:
        out = torch.empty(n_rows, (n_cols + 31) // 32, dtype=torch.int32, device=indptr.device)
    _lib.call("svg_lists_to_bitmap", n_rows, int(n_cols), indptr.data_ptr(), indices.data_ptr(),
              out.data_ptr(), _ptr(status), _stream(stream))
    return out


# --------------------------------------------------------------------- layer

class LayerBuffers:
    """Preallocated buffers for svg_layer at one shape (reused across steps)."""

    def __init__(self, q: torch.Tensor, S: int, layout: int = _lib.SVG_FUSE_OUTPUT,
                 qk: bool = False):
        B, H, N, d = q.shape
        dev = q.device
        if qk:  # q and k after QK-Norm + RoPE
            self.qn = torch.empty_like(q)
            self.kn = torch.empty_like(q)
        if not layout & _lib.SVG_FUSE_INPUT:  # token-major copies of q, k, v
            self.qp = torch.empty_like(q)
            self.kp = torch.empty_like(q)
            self.vp = torch.empty_like(q)
            # the V exponents run on this stream beside the profiling
            self.side = torch.cuda.Stream(device=dev) if dev.type == "cuda" else None
        if not layout & _lib.SVG_FUSE_OUTPUT:  # token-major output
            self.op = torch.empty_like(q)
        self.o = torch.empty_like(q)
        # per-head V exponents (svg_v_exponents) for the fp16 P.V product
        self.vexp = torch.empty(B * H, dtype=torch.int32, device=dev)
        self.mse = torch.empty(B * H, 2, dtype=torch.float32, device=dev)
        self.mode = torch.empty(B * H, dtype=torch.int32, device=dev)
        self.ws = _scratch(_lib.lib.svg_profile_workspace_size(B, H, N, d, S), dev)


def svg_layer(q, k, v, frames: int, tokens_per_frame: int, spatial_width: int,
              sample_idx: torch.Tensor, lists: BlockLists, bufs: Optional[LayerBuffers] = None,
              stream=None, layout: int = _lib.SVG_FUSE_OUTPUT, overlap: bool = True,
              qk: Optional[QKTransform] = None, repeat: Optional[torch.Tensor] = None,
              frame_shape: Optional[Sequence[int]] = None, anchors: int = 5):
    """One attention layer: profile -> block-sparse attention on the list the
    mode selects, temporal heads in token-major order.  `layout` picks which
    side of the reordering runs inside the attention kernel
    (svg_sparse_attn_fused); the other side runs as permutation kernels.
    The default fuses only the output side: on B200 the permutation kernel
    moves q, k, v faster than row gathers inside the attention kernel.  With
    overlap (input side not fused), the V exponents are computed on a side
    stream while the heads are profiled, and the token-major copies of the
    temporal heads alone follow the profiling (svg_permute_temporal_heads):
    the profiling kernel occupies every SM, so copies of every head beside it
    cost more than the copies the modes call for after it.
    qk applies QK-Norm + RoPE to q and k first (svg_qk_norm_rope); with
    overlap that pass also writes the token-major copies of q and k, and only
    v is copied after the profiling.
    repeat (int32 [B*H], nonzero = spatially repeating head, e.g. from
    svg_row_similarity > 0.87) with frame_shape = (rows, cols): those heads,
    unless profiled temporal, compute only the query tiles holding anchor
    rows and take the anchors' outputs on the other rows.
    Every bf16 layer also computes the per-head V exponents
    (svg_v_exponents), so any finite V stays exact in the fp16 P.V product.
    Returns (o, mode, mse)."""
    if bufs is None:
        bufs = LayerBuffers(q, sample_idx.numel(), layout, qk=qk is not None)
    if qk is not None and not hasattr(bufs, "qn"):
        raise ValueError("QK-Norm + RoPE needs LayerBuffers(..., qk=True)")
    F, P = frames, tokens_per_frame
    if repeat is not None and (frame_shape is None or frame_shape[0] * frame_shape[1] != P):
        raise ValueError("repeat needs frame_shape = (rows, cols) with rows * cols = P")

    def select_lists(st):
        """The lists and per-head ids the attention runs with (anchor lists
        are built once per buffers, lists and frame shape)."""
        if repeat is None:
            return lists, bufs.mode
        key = (lists.indptr.data_ptr(), lists.indices.data_ptr(), tuple(frame_shape), anchors)
        cached = getattr(bufs, "anchor_lists", None)
        if cached is None or cached[0] != key:
            alists, _ = svg_anchor_lists(lists, q.shape[2], F, frame_shape[0], frame_shape[1],
                                         anchors=anchors, stream=st)
            bufs.anchor_lists = cached = (key, alists, torch.empty_like(bufs.mode))
        _, alists, ids = cached
        svg_anchor_list_ids(bufs.mode, repeat, lists.n_lists, skip_list=SVG_MODE_TEMPORAL,
                            out=ids, stream=st)
        return alists, ids

    def broadcast(ids, st):
        if repeat is not None:
            svg_row_broadcast(bufs.o, F, frame_shape[0], frame_shape[1], ids, lists.n_lists,
                              anchors=anchors, stream=st)
    if overlap and not layout & _lib.SVG_FUSE_INPUT:
        # V exponents on a side stream beside the profiling; then token-major
        # copies of the temporal heads, which the attention reads for them
        if stream is None:
            main = torch.cuda.current_stream()
        elif hasattr(stream, "wait_event"):
            main = stream
        else:  # a raw cudaStream_t handle
            main = torch.cuda.ExternalStream(int(stream), device=q.device)
        ready = torch.cuda.Event()
        ready.record(main)
        bufs.side.wait_event(ready)
        if v.dtype == torch.bfloat16:
            svg_v_exponents(v, out=bufs.vexp, stream=bufs.side)
        side_done = torch.cuda.Event()
        side_done.record(bufs.side)
        if qk is not None:
            svg_qk_norm_rope(q, k, qk, out=(bufs.qn, bufs.kn), tm_out=(bufs.qp, bufs.kp),
                             frames=F, tokens_per_frame=P, stream=main)
            q, k = bufs.qn, bufs.kn
        svg_profile_heads(q, k, v, F, P, spatial_width, sample_idx, mse_out=bufs.mse,
                          mode_out=bufs.mode, workspace=bufs.ws, stream=main)
        copy_work = ((v, bufs.vp),) if qk is not None else \
            ((q, bufs.qp), (k, bufs.kp), (v, bufs.vp))
        for x, y in copy_work:
            svg_permute_temporal_heads(x, F, P, bufs.mode, out=y, stream=main)
        main.wait_event(side_done)
        bufs.vexp.record_stream(bufs.side)
        out = bufs.o if layout & _lib.SVG_FUSE_OUTPUT else bufs.op
        use_lists, ids = select_lists(main)
        svg_sparse_attn_fused(q, k, v, F, P, ids, use_lists, layout=layout,
                              copies=(bufs.qp, bufs.kp, bufs.vp), out=out, stream=main,
                              v_exp=bufs.vexp if v.dtype == torch.bfloat16 else None)
        if not layout & _lib.SVG_FUSE_OUTPUT:
            svg_permute_frame_major(bufs.op, F, P, bufs.mode, out=bufs.o, stream=main)
        broadcast(ids, main)
        return bufs.o, bufs.mode, bufs.mse
    if qk is not None:
        svg_qk_norm_rope(q, k, qk, out=(bufs.qn, bufs.kn), stream=stream)
        q, k = bufs.qn, bufs.kn
    svg_profile_heads(q, k, v, F, P, spatial_width, sample_idx, mse_out=bufs.mse,
                      mode_out=bufs.mode, workspace=bufs.ws, stream=stream)
    if layout & _lib.SVG_FUSE_INPUT:
        ins = (q, k, v)
    else:
        for x, y in ((q, bufs.qp), (k, bufs.kp), (v, bufs.vp)):
            svg_permute_token_major(x, F, P, bufs.mode, out=y, stream=stream)
        ins = (bufs.qp, bufs.kp, bufs.vp)
    use_lists, ids = select_lists(stream)
    vexp = None
    if v.dtype == torch.bfloat16:
        vexp = svg_v_exponents(v, out=bufs.vexp, stream=stream)
    if layout & _lib.SVG_FUSE_OUTPUT:
        svg_sparse_attn_fused(*ins, F, P, ids, use_lists, layout=layout, out=bufs.o,
                              stream=stream, v_exp=vexp)
    else:
        svg_sparse_attn_fused(*ins, F, P, ids, use_lists, layout=layout, out=bufs.op,
                              stream=stream, v_exp=vexp)
        svg_permute_frame_major(bufs.op, F, P, bufs.mode, out=bufs.o, stream=stream)
    broadcast(ids, stream)
    return bufs.o, bufs.mode, bufs.mse


class HostLayerBuffers:
    """Device slots for svg_layer_from_host: two chunks of `heads` heads each
    (inputs and LayerBuffers), and the copy streams."""

    def __init__(self, heads: int, N: int, d: int, S: int, device=None):
        dev = torch.device(device) if device is not None else torch.device("cuda")
        self.heads = heads
        self.slots = []
        for _ in range(2):
            x = torch.empty(3, 1, heads, N, d, dtype=torch.bfloat16, device=dev)
            slot = {"q": x[0], "k": x[1], "v": x[2], "bufs": LayerBuffers(x[0], S),
                    "loaded": torch.cuda.Event(), "computed": torch.cuda.Event(),
                    "unloaded": torch.cuda.Event(), "used": False}
            self.slots.append(slot)
        self.h2d = torch.cuda.Stream(device=dev)
        self.d2h = torch.cuda.Stream(device=dev)


def svg_layer_from_host(q, k, v, frames: int, tokens_per_frame: int, spatial_width: int,
                        sample_idx: torch.Tensor, lists: BlockLists, *, out=None, mode_out=None,
                        heads_per_chunk: int = 4, buffers: Optional[HostLayerBuffers] = None,
                        stream=None):
    """svg_layer for q, k, v in pinned host memory ([B, H, N, d] bf16): the
    B*H heads go through the GPU in chunks of `heads_per_chunk` (a divisor of
    B*H) on two device slots, so that the copy of chunk c + 1 to the device
    and of chunk c - 1 back to the host run while chunk c is computed (heads
    are independent in every step of the layer).  Returns (out, mode_out):
    pinned host [B, H, N, d] bf16 and [B*H] int32, complete once `stream`
    (default: the current stream) has passed this call."""
    B, H, N, d = q.shape
    BH = B * H
    for x in (q, k, v):
        if x.device.type != "cpu" or not x.is_pinned() or x.dtype != torch.bfloat16 \
                or not x.is_contiguous() or x.shape != q.shape:
            raise ValueError("svg_layer_from_host takes contiguous pinned host bf16 [B, H, N, d]")
    if heads_per_chunk <= 0 or BH % heads_per_chunk:
        raise ValueError(f"heads_per_chunk must divide B*H = {BH}")
    hc = heads_per_chunk
    dev = sample_idx.device
    if buffers is None or buffers.heads != hc or buffers.slots[0]["q"].shape[2:] != (N, d):
        buffers = HostLayerBuffers(hc, N, d, sample_idx.numel(), dev)
    if out is None:
        out = torch.empty(q.shape, dtype=torch.bfloat16).pin_memory()
    if mode_out is None:
        mode_out = torch.empty(BH, dtype=torch.int32).pin_memory()
    main = torch.cuda.current_stream(dev) if stream is None else stream
    qf, kf, vf, of = (x.view(BH, N, d) for x in (q, k, v, out))
    for c in range(BH // hc):
        slot = buffers.slots[c % 2]
        lo, hi = c * hc, (c + 1) * hc
        # inputs of chunk c once chunk c - 2 has been computed from this slot
        if slot["used"]:
            buffers.h2d.wait_event(slot["computed"])
        with torch.cuda.stream(buffers.h2d):
            for src, dst in ((qf, slot["q"]), (kf, slot["k"]), (vf, slot["v"])):
                dst[0].copy_(src[lo:hi], non_blocking=True)
        slot["loaded"].record(buffers.h2d)
        main.wait_event(slot["loaded"])
        if slot["used"]:  # the slot's output has gone back to the host
            main.wait_event(slot["unloaded"])
        o, mode, _ = svg_layer(slot["q"], slot["k"], slot["v"], frames, tokens_per_frame,
                               spatial_width, sample_idx, lists, slot["bufs"], stream=main)
        slot["computed"].record(main)
        buffers.d2h.wait_event(slot["computed"])
        with torch.cuda.stream(buffers.d2h):
            of[lo:hi].copy_(o[0], non_blocking=True)
            mode_out[lo:hi].copy_(mode, non_blocking=True)
        slot["unloaded"].record(buffers.d2h)
        slot["used"] = True
    for slot in buffers.slots:
        if slot["used"]:
            main.wait_event(slot["unloaded"])
    return out, mode_out


def svg_attention_from_host(q, k, v, list_id: torch.Tensor, lists: BlockLists, *, out=None,
                            heads_per_chunk: int = 4, buffers: Optional[HostLayerBuffers] = None,
                            stream=None):
    """Block-sparse attention (V exponents, then every head on its list:
    svg_v_exponents + svg_sparse_attn_fused with the lists' tile order) for
    q, k, v in pinned host memory ([B, H, N, d] bf16), streamed like
    svg_layer_from_host: chunks of `heads_per_chunk` heads (a divisor of B*H)
    through two device slots, the copies in and out overlapping the compute.
    list_id: device int32 [B*H].  Returns out (pinned host), complete once
    `stream` (default: the current stream) has passed this call."""
    B, H, N, d = q.shape
    BH = B * H
    for x in (q, k, v):
        if x.device.type != "cpu" or not x.is_pinned() or x.dtype != torch.bfloat16 \
                or not x.is_contiguous() or x.shape != q.shape:
            raise ValueError("svg_attention_from_host takes contiguous pinned host bf16 [B, H, N, d]")
    if heads_per_chunk <= 0 or BH % heads_per_chunk:
        raise ValueError(f"heads_per_chunk must divide B*H = {BH}")
    if list_id.numel() != BH or list_id.dtype != torch.int32:
        raise ValueError("list_id must be int32 [B*H]")
    hc = heads_per_chunk
    dev = list_id.device
    if buffers is None or buffers.heads != hc or buffers.slots[0]["q"].shape[2:] != (N, d):
        buffers = HostLayerBuffers(hc, N, d, 1, dev)
    if out is None:
        out = torch.empty(q.shape, dtype=torch.bfloat16).pin_memory()
    main = torch.cuda.current_stream(dev) if stream is None else stream
    qf, kf, vf, of = (x.view(BH, N, d) for x in (q, k, v, out))
    for c in range(BH // hc):
        slot = buffers.slots[c % 2]
        lo, hi = c * hc, (c + 1) * hc
        if slot["used"]:
            buffers.h2d.wait_event(slot["computed"])
        with torch.cuda.stream(buffers.h2d):
            for src, dst in ((qf, slot["q"]), (kf, slot["k"]), (vf, slot["v"])):
                dst[0].copy_(src[lo:hi], non_blocking=True)
        slot["loaded"].record(buffers.h2d)
        main.wait_event(slot["loaded"])
        if slot["used"]:
            main.wait_event(slot["unloaded"])
        bufs = slot["bufs"]
        vexp = svg_v_exponents(slot["v"], out=bufs.vexp, stream=main)
        o = svg_sparse_attn_fused(slot["q"], slot["k"], slot["v"], 1, N, list_id[lo:hi], lists,
                                  layout=0, out=bufs.o, v_exp=vexp, stream=main)
        slot["computed"].record(main)
        buffers.d2h.wait_event(slot["computed"])
        with torch.cuda.stream(buffers.d2h):
            of[lo:hi].copy_(o[0], non_blocking=True)
        slot["unloaded"].record(buffers.d2h)
        slot["used"] = True
    for slot in buffers.slots:
        if slot["used"]:
            main.wait_event(slot["unloaded"])
    return out
