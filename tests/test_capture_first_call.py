"""The attention launchers size their clusters lazily (occupancy queries
cached per device and kernel).  A process whose first call of a kernel is
made while a CUDA graph is being captured must still get a valid launch:
run in a fresh interpreter (cold caches), capture the first call of each
kernel family, replay it and compare with an eager call bit for bit."""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

SCRIPT = r'''
import sys
sys.path.insert(0, sys.argv[1])
import torch
from rotated_int4_kv_kvq_b200 import kvq, workloads as W
dev = torch.device("cuda", 0)
gen = torch.Generator(device=dev).manual_seed(5)
# tensor-core kernel with two query groups, the lane-pair kernel, the
# warp-per-token kernel (g < d), the tensor-core kernel with 4 queries
for d, g, nq, h, n in ((128, 128, 6, 3, 700), (64, 64, 1, 5, 900), (256, 64, 4, 2, 500),
                       (256, 256, 4, 9, 300)):
    signs = torch.from_numpy(W.make_signs(d)).to(dev)
    c = []
    for _ in range(2):
        x = torch.randn((h * n, d), generator=gen, device=dev).half()
        p, s = kvq.kvq_rot_quant_fwd(x, signs, 1, g)
        c += [p.reshape(h, n, -1), s.reshape(h, n, -1)]
    q = torch.randn((h, nq, d), generator=gen, device=dev).half()
    o = torch.empty((h, nq, d), dtype=torch.float16, device=dev)
    torch.cuda.synchronize()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.stream(side):
        with torch.cuda.graph(graph, stream=side):
            kvq.kvq_attend_decode(q, c[0], c[1], c[2], c[3], n, signs, 1, g, out=o)
    torch.cuda.current_stream().wait_stream(side)
    graph.replay()
    torch.cuda.synchronize()
    ref = kvq.kvq_attend_decode(q, c[0], c[1], c[2], c[3], n, signs, 1, g)
    torch.cuda.synchronize()
    assert torch.equal(o, ref), (d, g, nq)
    del graph
assert kvq.kvq_device_status() == 0
print("ok")
'''


def test_first_attention_call_inside_graph_capture():
    r = subprocess.run([sys.executable, "-c", SCRIPT, ROOT], capture_output=True, text=True,
                       timeout=600)
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-2000:]
    assert r.stdout.strip().endswith("ok")
