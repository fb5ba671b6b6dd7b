"""moe_route_dispatch against moe_route followed by moe_permute (x_perm NULL).

The one call must give exactly the outputs of the two: the selection, gates,
counts, n_ffn, probabilities and their column sums, and the dispatch layout.
The shapes cover each way the call runs: one cluster holding every token
group (T <= 16 at d = 2048; many groups at small d), one group (T <= 8), one
cluster per group with the ticket (decode T = 64 and 256), and the two-call
path (T > 256, and N too large for the layout tables in shared memory)."""
import pytest
import torch

from mixture_experts_layer_30_b200 import binding as B

pytestmark = pytest.mark.gpu


def _inputs(T, d, N, Z, dtype, seed, bias=None):
    g = torch.Generator(device="cpu").manual_seed(seed)
    dt = torch.float32 if dtype == "f32" else torch.bfloat16
    E = N + Z
    x = torch.randn((T, d), generator=g).to(dt).cuda()
    w = (torch.randn((E, d), generator=g) * 0.1).to(dt).cuda()
    b = (torch.rand(E, generator=g) * 0.1 - 0.05) if bias is None else torch.as_tensor(bias)
    return x, w, b.float().cuda()


def _outputs(shape, with_probs):
    T, K, E, N = shape.T, shape.K, shape.N + shape.Z, shape.N
    i32 = dict(dtype=torch.int32, device="cuda")
    o = dict(idx=torch.full((T, K), -7, **i32), gate=torch.full((T, K), -7.0, device="cuda"),
             counts=torch.full((E,), -7, **i32),
             n_ffn=torch.full((T,), 255, dtype=torch.uint8, device="cuda"),
             offsets=torch.full((N + 1,), -7, **i32), row_token=torch.full((T * K,), -7, **i32),
             slot_pos=torch.full((T, K), -7, **i32))
    if with_probs:
        o["probs"] = torch.full((T, E), -7.0, device="cuda")
        o["psum"] = torch.full((E,), -7.0, device="cuda")
    else:
        o["probs"] = o["psum"] = None
    return o


@pytest.mark.parametrize("T,d,N,Z,K,dtype", [
    (16, 2048, 64, 32, 6, "bf16"),   # one cluster of 8 x 2 CTAs
    (5, 2048, 64, 32, 6, "bf16"),    # one token group
    (64, 2048, 64, 32, 6, "bf16"),   # eight clusters, ticket
    (256, 2048, 64, 32, 6, "bf16"),  # 32 clusters, ticket
    (90, 64, 1, 2, 1, "f32"),        # one cluster of 1 x 12 CTAs
    (200, 128, 12, 4, 3, "f32"),     # 25 clusters, ticket
    (300, 128, 12, 4, 3, "bf16"),    # T > 256: the two-call path
    (150, 128, 640, 384, 40, "f32"),  # N > 481: the two-call path
])
@pytest.mark.parametrize("with_probs", [False, True])
def test_route_dispatch_equals_route_then_permute(T, d, N, Z, K, dtype, with_probs):
    shape = B.make_shape(T, d, N, Z, K, 64, dtype)
    x, w, bias = _inputs(T, d, N, Z, dtype, seed=T + N)
    ws = B.new_workspace(shape)
    a, b = _outputs(shape, with_probs), _outputs(shape, with_probs)
    B.route(shape, x, w, bias, ws, a["idx"], a["gate"], a["counts"], a["n_ffn"],
            probs_out=a["probs"], prob_sum=a["psum"])
    B.permute(shape, None, a["idx"], a["counts"], a["offsets"], a["row_token"], a["slot_pos"],
              None, ws)
    B.route_dispatch(shape, x, w, bias, ws, b["idx"], b["gate"], b["counts"], b["n_ffn"],
                     b["offsets"], b["row_token"], b["slot_pos"], probs_out=b["probs"],
                     prob_sum=b["psum"])
    torch.cuda.synchronize()
    assert B.device_status(ws) == 0
    R = int(a["offsets"][-1])
    assert R > 0
    for k in ("idx", "gate", "counts", "n_ffn", "offsets", "slot_pos") + (
            ("probs", "psum") if with_probs else ()):
        assert torch.equal(a[k], b[k]), k
    assert torch.equal(a["row_token"][:R], b["row_token"][:R])


def test_route_dispatch_all_slots_to_zero_experts():
    """Every slot on a zero-computation expert: no rows, offsets all 0."""
    N, Z, K = 16, 8, 4
    shape = B.make_shape(32, 256, N, Z, K, 64, "bf16")
    x, w, bias = _inputs(32, 256, N, Z, "bf16", seed=3, bias=[0.0] * N + [10.0] * Z)
    ws = B.new_workspace(shape)
    o = _outputs(shape, False)
    B.route_dispatch(shape, x, w, bias, ws, o["idx"], o["gate"], o["counts"], o["n_ffn"],
                     o["offsets"], o["row_token"], o["slot_pos"])
    torch.cuda.synchronize()
    assert B.device_status(ws) == 0
    assert (o["idx"] >= N).all()
    assert int(o["n_ffn"].sum()) == 0
    assert (o["offsets"] == 0).all()
    assert (o["slot_pos"] == -1).all()
