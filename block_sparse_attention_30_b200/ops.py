"""Python front-end with the C ABI's names: torch tensors in, kernel launches
out.  PyTorch supplies device memory and the current stream; each function
only checks dtypes/shapes and forwards raw pointers to libvsa.so.
"""
import torch

from . import _lib

_SENTINEL = object()


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return s.cuda_stream


def _ptr(t):
    return None if t is None else t.data_ptr()


def _shape(B, heads, head_dim, T, H, W, tile):
    tt, th, tw = tile
    return [B, heads, head_dim, T, H, W, tt, th, tw]


def _grid_of(x, T, H, W):
    assert x.dim() == 4 and x.is_contiguous(), "expected a contiguous [B, N, heads, d] tensor"
    B, N, heads, d = x.shape
    assert N == T * H * W, f"N={N} does not match grid {T}x{H}x{W}"
    return B, heads, d


def vsa_status_string(code: int) -> str:
    return _lib.lib().vsa_status_string(code).decode()


def vsa_num_tiles(T, H, W, tile=(4, 4, 4)) -> int:
    return _lib.lib().vsa_num_tiles(T, H, W, *tile)


def vsa_workspace_bytes(B, heads, head_dim, T, H, W, topk, tile=(4, 4, 4)) -> int:
    return _lib.lib().vsa_workspace_bytes(*_shape(B, heads, head_dim, T, H, W, tile), topk)


def new_workspace(B, heads, head_dim, T, H, W, topk, tile=(4, 4, 4), device="cuda", stream=None):
    """Allocate (torch) and initialise a workspace for these shapes."""
    n = vsa_workspace_bytes(B, heads, head_dim, T, H, W, topk, tile)
    if n == 0:
        raise _lib.VSAError("vsa_workspace_bytes", 1)
    ws = torch.empty(n, dtype=torch.uint8, device=device)
    _lib.check("vsa_workspace_init", _lib.lib().vsa_workspace_init(ws.data_ptr(), n, _stream(stream)))
    return ws


def vsa_gather_tiles(x, x_tiles, T, H, W, tile=(4, 4, 4), stream=None):
    B, heads, d = _grid_of(x, T, H, W)
    _lib.check("vsa_gather_tiles", _lib.lib().vsa_gather_tiles(
        x.data_ptr(), x_tiles.data_ptr(), *_shape(B, heads, d, T, H, W, tile), _stream(stream)))


def vsa_scatter_tiles(x_tiles, x, T, H, W, tile=(4, 4, 4), stream=None):
    B, heads, d = _grid_of(x, T, H, W)
    _lib.check("vsa_scatter_tiles", _lib.lib().vsa_scatter_tiles(
        x_tiles.data_ptr(), x.data_ptr(), *_shape(B, heads, d, T, H, W, tile), _stream(stream)))


def vsa_select_blocks(q, k, T, H, W, topk, block_idx, workspace, tile=(4, 4, 4), stream=None):
    B, heads, d = _grid_of(q, T, H, W)
    _lib.check("vsa_select_blocks", _lib.lib().vsa_select_blocks(
        q.data_ptr(), k.data_ptr(), *_shape(B, heads, d, T, H, W, tile), topk,
        block_idx.data_ptr(), workspace.data_ptr(), workspace.numel(), _stream(stream)))


def vsa_select_blocks_noalloc(q, k, T, H, W, topk, block_idx, tile=(4, 4, 4), stream=None):
    """vsa_select_blocks without a workspace: for callers that cannot allocate
    device memory.  The library's fixed device array holds the intermediates."""
    B, heads, d = _grid_of(q, T, H, W)
    _lib.check("vsa_select_blocks_noalloc", _lib.lib().vsa_select_blocks_noalloc(
        q.data_ptr(), k.data_ptr(), *_shape(B, heads, d, T, H, W, tile), topk,
        block_idx.data_ptr(), _stream(stream)))


def vsa_linear_branch_fwd(k, v, lin_S, lin_z, T, H, W, workspace, stream=None):
    B, heads, d = _grid_of(k, T, H, W)
    _lib.check("vsa_linear_branch_fwd", _lib.lib().vsa_linear_branch_fwd(
        k.data_ptr(), v.data_ptr(), lin_S.data_ptr(), lin_z.data_ptr(), B, heads, d, T, H, W,
        workspace.data_ptr(), workspace.numel(), _stream(stream)))


def vsa_sparse_attn_fwd(q, k, v, block_idx, out, T, H, W, topk, workspace, lin_S=None, lin_z=None,
                        tile=(4, 4, 4), stream=None):
    B, heads, d = _grid_of(q, T, H, W)
    _lib.check("vsa_sparse_attn_fwd", _lib.lib().vsa_sparse_attn_fwd(
        q.data_ptr(), k.data_ptr(), v.data_ptr(), block_idx.data_ptr(), _ptr(lin_S), _ptr(lin_z),
        out.data_ptr(), *_shape(B, heads, d, T, H, W, tile), topk, workspace.data_ptr(),
        workspace.numel(), _stream(stream)))


def vsa_sparse_attn_fwd_train(q, k, v, block_idx, out, out_f32, lse, T, H, W, topk, workspace,
                              tile=(4, 4, 4), stream=None):
    """Sparse-branch forward that also writes, for the backward pass, an fp32
    copy of the output and lse[B][heads][nt][64] (fp32)."""
    B, heads, d = _grid_of(q, T, H, W)
    _lib.check("vsa_sparse_attn_fwd_train", _lib.lib().vsa_sparse_attn_fwd_train(
        q.data_ptr(), k.data_ptr(), v.data_ptr(), block_idx.data_ptr(), out.data_ptr(),
        out_f32.data_ptr(), lse.data_ptr(), *_shape(B, heads, d, T, H, W, tile), topk,
        workspace.data_ptr(), workspace.numel(), _stream(stream)))


def vsa_sparse_attn_bwd(q, k, v, out_f32, dout, block_idx, lse, dq, dk, dv, T, H, W, topk, workspace,
                        tile=(4, 4, 4), stream=None):
    """Gradients dq, dk, dv (bf16, written in place) of the fine pass."""
    B, heads, d = _grid_of(q, T, H, W)
    _lib.check("vsa_sparse_attn_bwd", _lib.lib().vsa_sparse_attn_bwd(
        q.data_ptr(), k.data_ptr(), v.data_ptr(), out_f32.data_ptr(), dout.data_ptr(),
        block_idx.data_ptr(), lse.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(),
        *_shape(B, heads, d, T, H, W, tile), topk, workspace.data_ptr(), workspace.numel(),
        _stream(stream)))


def vsa_linear_branch_bwd(q, k, v, dout, lin_S, lin_z, dq, dk, dv, T, H, W, workspace,
                          accumulate=False, stream=None):
    """Gradients dq, dk, dv (bf16, in place) of the linear branch
    phi(q)S/(phi(q).z); with accumulate=True they are added to the values
    already in dq, dk, dv."""
    B, heads, d = _grid_of(q, T, H, W)
    _lib.check("vsa_linear_branch_bwd", _lib.lib().vsa_linear_branch_bwd(
        q.data_ptr(), k.data_ptr(), v.data_ptr(), dout.data_ptr(), lin_S.data_ptr(),
        lin_z.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), int(bool(accumulate)), B,
        heads, d, T, H, W, workspace.data_ptr(), workspace.numel(), _stream(stream)))


def vsa_quantize_qk_e4m3(q, k, q8, k8, q_scale, k_scale, T, H, W, tile=(4, 4, 4), stream=None):
    """Per-cube E4M3 codes (uint8, q's layout) and fp32 scales [B, heads, nt]
    of q and k, written in place."""
    B, heads, d = _grid_of(q, T, H, W)
    _lib.check("vsa_quantize_qk_e4m3", _lib.lib().vsa_quantize_qk_e4m3(
        q.data_ptr(), k.data_ptr(), q8.data_ptr(), k8.data_ptr(), q_scale.data_ptr(),
        k_scale.data_ptr(), *_shape(B, heads, d, T, H, W, tile), _stream(stream)))


def vsa_sparse_attn_fwd_e4m3(q8, k8, q_scale, k_scale, v, block_idx, out, T, H, W, topk, workspace,
                             tile=(4, 4, 4), stream=None):
    """Fine pass with Q K^T in E4M3 (codes and scales from vsa_quantize_qk_e4m3)."""
    B, heads, d = _grid_of(v, T, H, W)
    _lib.check("vsa_sparse_attn_fwd_e4m3", _lib.lib().vsa_sparse_attn_fwd_e4m3(
        q8.data_ptr(), k8.data_ptr(), q_scale.data_ptr(), k_scale.data_ptr(), v.data_ptr(),
        block_idx.data_ptr(), out.data_ptr(), *_shape(B, heads, d, T, H, W, tile), topk,
        workspace.data_ptr(), workspace.numel(), _stream(stream)))


def vsa_sparse_linear_attn_fwd_e4m3(q8, k8, q_scale, k_scale, q, v, block_idx, lin_S, lin_z, out, T, H,
                                    W, topk, workspace, tile=(4, 4, 4), stream=None):
    """Fine pass with Q K^T in E4M3 plus the bf16 linear branch phi(q)S/(phi(q).z)
    (lin_S, lin_z from vsa_linear_branch_fwd)."""
    B, heads, d = _grid_of(v, T, H, W)
    _lib.check("vsa_sparse_linear_attn_fwd_e4m3", _lib.lib().vsa_sparse_linear_attn_fwd_e4m3(
        q8.data_ptr(), k8.data_ptr(), q_scale.data_ptr(), k_scale.data_ptr(), q.data_ptr(),
        v.data_ptr(), block_idx.data_ptr(), lin_S.data_ptr(), lin_z.data_ptr(), out.data_ptr(),
        *_shape(B, heads, d, T, H, W, tile), topk, workspace.data_ptr(), workspace.numel(),
        _stream(stream)))


def vsa_device_status(workspace, stream=None) -> int:
    """Synchronise and return the device status code (0 = VSA_OK)."""
    return _lib.lib().vsa_device_status(workspace.data_ptr(), _stream(stream))


class BlockSparseVideoAttention:
    """Whole forward pass for one grid shape: select -> (linear state) -> fine.

    Buffers (indices, linear state, workspace) are allocated once by torch and
    reused by every call; `__call__` only enqueues kernels on the stream.
    """

    def __init__(self, B, heads, head_dim, T, H, W, topk, tile=(4, 4, 4), linear=False,
                 device="cuda"):
        self.shape = (B, heads, head_dim, T, H, W)
        self.T, self.H, self.W, self.topk, self.tile, self.linear = T, H, W, topk, tuple(tile), linear
        nt = vsa_num_tiles(T, H, W, tile)
        self.num_tiles = nt
        self.block_idx = torch.empty((B, heads, nt, topk), dtype=torch.int32, device=device)
        self.workspace = new_workspace(B, heads, head_dim, T, H, W, topk, tile, device)
        if linear:
            self.lin_S = torch.empty((B, heads, head_dim, head_dim), dtype=torch.float32, device=device)
            self.lin_z = torch.empty((B, heads, head_dim), dtype=torch.float32, device=device)
        else:
            self.lin_S = self.lin_z = None

    def __call__(self, q, k, v, out=None, stream=None):
        for x in (q, k, v):
            assert x.dtype == torch.bfloat16 and x.is_cuda and tuple(x.shape[1:]) == (
                self.T * self.H * self.W, self.shape[1], self.shape[2])
        if out is None:
            out = torch.empty_like(q)
        vsa_select_blocks(q, k, self.T, self.H, self.W, self.topk, self.block_idx, self.workspace,
                          self.tile, stream)
        if self.linear:
            vsa_linear_branch_fwd(k, v, self.lin_S, self.lin_z, self.T, self.H, self.W,
                                  self.workspace, stream)
        vsa_sparse_attn_fwd(q, k, v, self.block_idx, out, self.T, self.H, self.W, self.topk,
                            self.workspace, self.lin_S, self.lin_z, self.tile, stream)
        return out

    def status(self, stream=None) -> int:
        return vsa_device_status(self.workspace, stream)


class HostPipeline:
    """Forward passes over a stream of host batches (pinned q, k, v in, output
    back to pinned host memory), with the copies overlapping the kernels.

    Two device buffer sets and three CUDA streams: while the kernels of step i
    run, the inputs of step i+1 travel host -> device and the output of step
    i-1 device -> host (the two copy directions use separate DMA engines).
    Events order each buffer set's reuse: inputs are overwritten only after
    the kernels that read them, outputs only after their copy back.
    """

    def __init__(self, attn, shape, dtype=torch.bfloat16, device="cuda"):
        self.attn = attn
        dev = torch.device(device)
        self.bufs = [tuple(torch.empty(shape, dtype=dtype, device=dev) for _ in range(4))
                     for _ in range(2)]                       # q, k, v, out per set
        self.s_in, self.s_comp, self.s_out = (torch.cuda.Stream(dev) for _ in range(3))
        self.ev_in = [torch.cuda.Event() for _ in range(2)]
        self.ev_comp = [torch.cuda.Event() for _ in range(2)]
        self.ev_out = [torch.cuda.Event() for _ in range(2)]
        self.used = [False, False]

    def run(self, items):
        """items: iterable of (q_h, k_h, v_h, out_h) pinned host tensors of the
        pipeline's shape.  Enqueues everything; call synchronize() (or wait on
        the returned event) before reading the host outputs."""
        for i, (qh, kh, vh, oh) in enumerate(items):
            x = i % 2
            q, k, v, o = self.bufs[x]
            with torch.cuda.stream(self.s_in):
                if self.used[x]:
                    self.s_in.wait_event(self.ev_comp[x])     # kernels of step i-2 read q, k, v
                q.copy_(qh, non_blocking=True)
                k.copy_(kh, non_blocking=True)
                v.copy_(vh, non_blocking=True)
                self.ev_in[x].record(self.s_in)
            self.s_comp.wait_event(self.ev_in[x])
            if self.used[x]:
                self.s_comp.wait_event(self.ev_out[x])        # output of step i-2 copied back
            self.attn(q, k, v, out=o, stream=self.s_comp)
            self.ev_comp[x].record(self.s_comp)
            with torch.cuda.stream(self.s_out):
                self.s_out.wait_event(self.ev_comp[x])
                oh.copy_(o, non_blocking=True)
                self.ev_out[x].record(self.s_out)
            self.used[x] = True
        done = torch.cuda.Event(enable_timing=True)
        done.record(self.s_out)
        return done

    def synchronize(self):
        for s in (self.s_in, self.s_comp, self.s_out):
            s.synchronize()
