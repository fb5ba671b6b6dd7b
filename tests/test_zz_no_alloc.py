"""moe_permute_noalloc against moe_permute.

The no-workspace dispatch serves callers that cannot hand the library any
scratch memory (operator plug-ins that only receive a call's input and output
buffers, runtimes that forbid allocations after start-up).  Its results must
be identical to the workspace version; two calls in a row with different
shapes and inputs check that nothing left in the shared scratch array leaks
into the next call.  This file is collected last on purpose.
"""
import ctypes

import pytest
import torch

from mixture_experts_layer_30_b200 import binding as B

pytestmark = pytest.mark.gpu

SCRATCH_BYTES = 4 << 20


def _scratch_bytes(T, N):
    tables = -(-T // 256) * N * 4
    return 256 + 2 * (-(-tables // 256) * 256)


def _routed(T, d, N, Z, K, I, dtype, seed):
    g = torch.Generator(device="cpu").manual_seed(seed)
    dt = torch.float32 if dtype == "f32" else torch.bfloat16
    x = torch.randn((T, d), generator=g).to(dt).cuda()
    w = (torch.randn((N + Z, d), generator=g) * 0.1).to(dt).cuda()
    bias = (torch.rand(N + Z, generator=g) * 0.1 - 0.05).cuda()
    shape = B.make_shape(T, d, N, Z, K, I, dtype)
    buf = B.LayerBuffers(shape)
    B.route(shape, x, w, bias, buf.ws, buf.topk_idx, buf.topk_gate, buf.counts, buf.n_ffn)
    return shape, x, buf


def _compare(shape, x, buf):
    B.permute(shape, x, buf.topk_idx, buf.counts, buf.offsets, buf.row_token, buf.slot_pos,
              buf.x_perm, buf.ws)
    offsets = torch.full_like(buf.offsets, -7)
    row_token = torch.full_like(buf.row_token, -7)
    slot_pos = torch.full_like(buf.slot_pos, -7)
    x_perm = torch.full_like(buf.x_perm, -7)
    B.permute_noalloc(shape, x, buf.topk_idx, buf.counts, offsets, row_token, slot_pos, x_perm)
    torch.cuda.synchronize()
    R = int(buf.offsets[-1])
    assert R > 0
    assert torch.equal(offsets, buf.offsets)
    assert torch.equal(row_token[:R], buf.row_token[:R])
    assert torch.equal(slot_pos, buf.slot_pos)
    assert torch.equal(x_perm[:R], buf.x_perm[:R])
    assert B.device_status(buf.ws) == 0


def test_noalloc_dispatch_matches_workspace_dispatch_twice():
    # multi-chunk layout (histogram, scan, rank): two calls in a row
    for T, d, N, Z, K, dtype, seed in ((700, 256, 64, 32, 6, "bf16", 1),
                                       (300, 128, 12, 4, 3, "f32", 2)):
        _compare(*_routed(T, d, N, Z, K, 64, dtype, seed))


def test_noalloc_decode_dispatch_matches_workspace_dispatch_twice():
    # batches of at most 256 tokens take the one-CTA layout path
    for T, d, N, Z, K, dtype, seed in ((64, 2048, 64, 32, 6, "bf16", 3),
                                       (16, 256, 16, 8, 4, "f32", 4)):
        _compare(*_routed(T, d, N, Z, K, 64, dtype, seed))


def test_noalloc_dispatch_at_its_largest_accepted_shape():
    # N = 1024: T = 130816 is the largest batch whose tables fit the 4 MiB array
    T, N, d = 130816, 1024, 8
    assert _scratch_bytes(T, N) <= SCRATCH_BYTES < _scratch_bytes(T + 1, N)
    g = torch.Generator(device="cpu").manual_seed(5)
    shape = B.make_shape(T, d, N, 0, 1, 64, "bf16")
    buf = B.LayerBuffers(shape)
    idx = torch.randint(0, N, (T, 1), generator=g, dtype=torch.int32)
    buf.topk_idx.copy_(idx)
    buf.counts.copy_(torch.bincount(idx.view(-1).long(), minlength=N).to(torch.int32))
    x = torch.randn((T, d), generator=g).to(torch.bfloat16).cuda()
    _compare(shape, x, buf)


def test_noalloc_dispatch_rejects_shapes_beyond_its_scratch():
    # one token past the limit at N = 1024: refused on the host before anything is
    # launched (the pointers are never dereferenced)
    fake = ctypes.c_void_p(256)
    for T, N in ((130817, 1024), (300_000, 1000)):
        assert _scratch_bytes(T, N) > SCRATCH_BYTES
        shape = B.make_shape(T, 64, N, 0, 1, 64, "f32")
        code = B.lib().moe_permute_noalloc(ctypes.byref(shape), fake, fake, None, fake, fake,
                                           fake, fake, None)
        assert code == 2  # MOE_ERR_UNSUPPORTED
        assert b"built-in array holds" in B.lib().moe_last_error()
