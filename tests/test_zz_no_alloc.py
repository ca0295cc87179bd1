"""The allocation-free selection entry point, vsa_select_blocks_noalloc.

It serves callers that cannot allocate device memory and therefore cannot hand
vsa_select_blocks a workspace; it keeps its intermediates in the library's
fixed device array instead.  This file is collected last on purpose, so a run
that stops at the first failure has already run every other test.  Checked
here: through the C ABI, two calls in a row on different inputs give the same
block indices as vsa_select_blocks (bit-exact: the same kernels run), and a
shape too large for the fixed array is refused before any work is enqueued.
"""
import ctypes

import pytest
import torch

from block_sparse_attention_30_b200 import WORKLOADS, _lib, build, synth

pytestmark = pytest.mark.gpu

VSA_OK, VSA_ERR_WORKSPACE = 0, 3


@pytest.fixture(scope="module")
def L():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    build.build()
    return _lib.lib()


def _select_both(L, w, seed):
    q, k, _ = synth.make_qkv(w.B, w.heads, w.head_dim, w.T, w.H, w.W, w.tile, w.amplitude, seed)
    q, k = q.cuda(), k.cuda()
    tt, th, tw = w.tile
    shape = (w.B, w.heads, w.head_dim, w.T, w.H, w.W, tt, th, tw)
    nt = L.vsa_num_tiles(w.T, w.H, w.W, tt, th, tw)
    stream = torch.cuda.current_stream().cuda_stream
    # existing entry point, with a torch-allocated workspace
    ws_bytes = L.vsa_workspace_bytes(*shape, w.topk)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")
    assert L.vsa_workspace_init(ws.data_ptr(), ws_bytes, stream) == VSA_OK
    ref = torch.full((w.B, w.heads, nt, w.topk), -1, dtype=torch.int32, device="cuda")
    assert L.vsa_select_blocks(q.data_ptr(), k.data_ptr(), *shape, w.topk, ref.data_ptr(),
                               ws.data_ptr(), ws_bytes, stream) == VSA_OK
    # allocation-free entry point
    got = torch.full_like(ref, -1)
    assert L.vsa_select_blocks_noalloc(q.data_ptr(), k.data_ptr(), *shape, w.topk,
                                       got.data_ptr(), stream) == VSA_OK
    torch.cuda.synchronize()
    return ref, got


def test_noalloc_select_matches_workspace_select_twice(L):
    w = WORKLOADS["wan1.3b_480p"]            # 21.6 MB of intermediates: fits the array
    for seed in (101, 202):                  # two calls in a row, different inputs
        ref, got = _select_both(L, w, seed)
        assert (ref >= 0).all()
        assert torch.equal(got, ref)


def test_noalloc_select_rejects_shapes_beyond_the_array(L):
    w = WORKLOADS["wan14b_480p"]             # 50 MB of intermediates: too large
    tt, th, tw = w.tile
    fake = 0x10000                           # never dereferenced: refused before launch
    code = L.vsa_select_blocks_noalloc(fake, fake, w.B, w.heads, w.head_dim, w.T, w.H, w.W,
                                       tt, th, tw, w.topk, fake, None)
    assert code == VSA_ERR_WORKSPACE
    assert _lib.NOALLOC_SELECT_SCRATCH_BYTES == 32 * 1024 * 1024
