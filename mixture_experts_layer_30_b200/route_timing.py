"""Times the route call alone: router GEMM + fp32 softmax + biased top-K + counts
(``moe_route``), the first step of the layer.

    python -m mixture_experts_layer_30_b200.route_timing WORKLOAD [WORKLOAD ...]

For each named workload of ``configs.CONFIGS`` it draws the layer's x, W_r and
bias (no expert weights, so the device holds a few hundred MB at most), calls
``moe_route`` 5 times as a warm-up, then times it with CUDA events:

- ``route_us_back_to_back``: 50 eager calls in a row (host launch cost included
  whenever it exceeds the kernels' time);
- ``route_us_graph``: one call captured in a CUDA graph, replayed 50 times (the
  graph's launch included in each);
- ``route_us_in_graph_of_50``: 50 calls captured in one graph, replayed 5 times
  (device time per call, consecutive calls overlapping through programmatic
  dependent launch).

One JSON object per workload is printed, with the workspace status word.
"""
import json
import sys

import torch

from . import binding as B
from . import configs as C
from . import inputs as IN


def time_route(cfg, n=50):
    L = IN.make_layer_inputs(cfg, device="cuda", with_experts=False)
    shape = B.shape_of(cfg)
    ws = B.new_workspace(shape)
    idx = torch.empty((cfg.T, cfg.K), dtype=torch.int32, device="cuda")
    gate = torch.empty((cfg.T, cfg.K), dtype=torch.float32, device="cuda")
    counts = torch.empty(cfg.E, dtype=torch.int32, device="cuda")
    nffn = torch.empty(cfg.T, dtype=torch.uint8, device="cuda")

    def call():
        B.route(shape, L["x"], L["w_router"], L["bias"], ws, idx, gate, counts, nffn)

    for _ in range(5):
        call()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(n):
        call()
    e1.record()
    torch.cuda.synchronize()
    back = e0.elapsed_time(e1) / n * 1e3
    g1 = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g1):
        call()
    g1.replay()
    torch.cuda.synchronize()
    e0.record()
    for _ in range(n):
        g1.replay()
    e1.record()
    torch.cuda.synchronize()
    one = e0.elapsed_time(e1) / n * 1e3
    gn = torch.cuda.CUDAGraph()
    with torch.cuda.graph(gn):
        for _ in range(n):
            call()
    gn.replay()
    torch.cuda.synchronize()
    e0.record()
    for _ in range(5):
        gn.replay()
    e1.record()
    torch.cuda.synchronize()
    many = e0.elapsed_time(e1) / (5 * n) * 1e3
    return {"workload": cfg.name, "route_us_back_to_back": round(back, 2),
            "route_us_graph": round(one, 2), "route_us_in_graph_of_50": round(many, 2),
            "status": B.device_status(ws)}


def main(argv):
    if not argv:
        print(__doc__)
        return 2
    for name in argv:
        print(json.dumps(time_route(C.CONFIGS[name])), flush=True)
        torch.cuda.empty_cache()
    return 0


if __name__ == "__main__":
    sys.exit(main(sys.argv[1:]))
