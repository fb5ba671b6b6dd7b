"""moe_permute_noalloc against moe_permute.

The no-workspace dispatch serves callers that cannot hand the library any
scratch memory (operator plug-ins that only receive a call's input and output
buffers, runtimes that forbid allocations after start-up).  Its results must
be identical to the workspace version; two calls in a row with different
shapes and inputs check that nothing left in the shared scratch array leaks
into the next call.  This file is collected last on purpose.
"""
import pytest
import torch

from mixture_experts_layer_30_b200 import binding as B

pytestmark = pytest.mark.gpu


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


def test_noalloc_dispatch_matches_workspace_dispatch_twice():
    for T, d, N, Z, K, dtype, seed in ((700, 256, 64, 32, 6, "bf16", 1),
                                       (300, 128, 12, 4, 3, "f32", 2)):
        shape, x, buf = _routed(T, d, N, Z, K, 64, dtype, seed)
        B.permute(shape, x, buf.topk_idx, buf.counts, buf.offsets, buf.row_token, buf.slot_pos,
                  buf.x_perm, buf.ws)
        offsets = torch.full_like(buf.offsets, -7)
        row_token = torch.full_like(buf.row_token, -7)
        slot_pos = torch.full_like(buf.slot_pos, -7)
        x_perm = torch.full_like(buf.x_perm, -7)
        B.permute_noalloc(shape, x, buf.topk_idx, buf.counts, offsets, row_token, slot_pos,
                          x_perm)
        torch.cuda.synchronize()
        R = int(buf.offsets[-1])
        assert R > 0
        assert torch.equal(offsets, buf.offsets)
        assert torch.equal(row_token[:R], buf.row_token[:R])
        assert torch.equal(slot_pos, buf.slot_pos)
        assert torch.equal(x_perm[:R], buf.x_perm[:R])
        assert B.device_status(buf.ws) == 0


def test_noalloc_dispatch_rejects_shapes_beyond_its_scratch():
    # 2 * ceil(T/256) * N * 4 + 512 bytes must fit in the 4 MiB array: T = 300000
    # tokens with N = 1000 experts needs about 9.4 MB, so the call is refused
    # before anything is launched (the pointers are never dereferenced).
    import ctypes
    shape = B.make_shape(300_000, 64, 1000, 0, 1, 64, "f32")
    fake = ctypes.c_void_p(256)
    code = B.lib().moe_permute_noalloc(ctypes.byref(shape), fake, fake, None, fake, fake, fake,
                                       fake, None)
    assert code == 2  # MOE_ERR_UNSUPPORTED
    assert b"built-in array holds" in B.lib().moe_last_error()
