"""The library's calls under CUDA graph capture: every call enqueues only
kernels and memsets on the caller's stream (no host synchronisation, no
allocation), so a sequence of calls can be captured once and replayed.  Each
case captures a call on a side stream (after one eager call there, which sizes
the workspace and the launch caches), replays the graph, and compares its
outputs bit for bit with an eager call on the same inputs (the kernels are
deterministic); it then changes the inputs in place and replays again."""
import numpy as np
import pytest
import torch

import oracle as O
from exact_laplace_b200 import laplex as X
from exact_laplace_b200 import synth
from gpu_util import assert_close, dev, host

pytestmark = pytest.mark.gpu


def capture(fn):
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        fn()  # eager on the capture stream: its workspace and the launch caches exist before capture
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        fn()
    return g


def bits_equal(a, b):
    a, b = host(a), host(b)
    return np.array_equal(a.view(np.uint8), b.view(np.uint8))


def refill(t, seed):
    t.copy_(torch.from_numpy(synth.normal(t.numel(), seed=seed, stream="x").reshape(t.shape)).to(t.device))


def test_graph_symmetric_products():
    n = 300_001
    a, x = synth.sym_uniform(n, 0.0, float(n), seed=1)
    s, perm = O.stable_sort(a)
    s_d, p_d, x_d = dev(s.astype(np.float32)), dev(perm.astype(np.int32)), dev(x)
    y_g = torch.empty_like(x_d)
    yb_g = torch.empty_like(x_d)
    g = capture(lambda: (X.matvec_sym(s_d, x_d, p_d, out=y_g), X.matvec_sym(s_d, x_d, out=yb_g)))
    for seed in (None, 7):
        if seed is not None:
            refill(x_d, seed)
        g.replay()
        torch.cuda.synchronize()
        assert bits_equal(y_g, X.matvec_sym(s_d, x_d, p_d))
        assert bits_equal(yb_g, X.matvec_sym(s_d, x_d))
    xh = host(x_d)
    assert_close(host(y_g), O.sym(a, xh), O.norm_sym(a, xh), np.float32, "graph replay", slack=O.far_mass(a, xh))


def test_graph_general_phased_gram_backward():
    n, k = 200_003, 50_001
    a, b, x, w = synth.general_ties(n, k, -100.0, 100.0, seed=2)
    sa = dev(np.sort(a).astype(np.float32))
    sb = dev(np.sort(b).astype(np.float32))
    xb, wa = dev(x), dev(w)
    phi = dev(synth.uniform(n, 0.0, 6.283, seed=2, stream="phi"))
    g_d = dev(synth.normal(n, seed=3, stream="g"))
    outs = {"Kx": torch.empty(n, device="cuda"), "KTw": torch.empty(k, device="cuda"),
            "phased": torch.empty(n, device="cuda"), "gram": torch.empty(n, device="cuda"),
            "dx": torch.empty(n, device="cuda"), "da": torch.empty(n, device="cuda")}

    def calls():
        X.matvec_general(sa, sb, xb, out=outs["Kx"])
        X.matvec_general(sa, sb, wa, transpose=True, out=outs["KTw"])
        X.matvec_phased(sa, phi, wa, out=outs["phased"])
        X.gram(sa, wa, phi=phi, out=outs["gram"])
        X.backward(sa, wa, g_d, dx_out=outs["dx"], da_out=outs["da"])

    gr = capture(calls)
    for seed in (None, 11):
        if seed is not None:
            refill(wa, seed)
        gr.replay()
        torch.cuda.synchronize()
        assert bits_equal(outs["Kx"], X.matvec_general(sa, sb, xb))
        assert bits_equal(outs["KTw"], X.matvec_general(sa, sb, wa, transpose=True))
        assert bits_equal(outs["phased"], X.matvec_phased(sa, phi, wa))
        assert bits_equal(outs["gram"], X.gram(sa, wa, phi=phi))
        dx, da = X.backward(sa, wa, g_d)
        assert bits_equal(outs["dx"], dx) and bits_equal(outs["da"], da)


def test_graph_sort_and_unsorted_product():
    """The sort, the carrying sort and the one-call product on unsorted anchors
    (digit passes, counts, permutation passes) replayed from one graph."""
    n = 1_000_003
    a, x = synth.sym_normal(n, 2000.0, B=1, seed=4)
    a_d, x_d = dev(a), dev(x)
    s1, p1 = torch.empty_like(a_d), torch.empty(n, dtype=torch.int32, device="cuda")
    s2, p2, xs2 = torch.empty_like(a_d), torch.empty(n, dtype=torch.int32, device="cuda"), torch.empty_like(x_d)
    y3, s3, p3 = torch.empty_like(x_d), torch.empty_like(a_d), torch.empty(n, dtype=torch.int32, device="cuda")

    def calls():
        X.sort_anchors(a_d, s1, p1)
        X.sort_anchors_carry(a_d, x_d, s2, p2, xs2)
        X.matvec_sym_unsorted(a_d, x_d, out=y3, sorted_out=s3, perm_out=p3)

    g = capture(calls)
    g.replay()
    torch.cuda.synchronize()
    _, ref = O.stable_sort(a)
    for p in (p1, p2, p3):
        assert np.array_equal(host(p), ref.astype(np.int32))
    assert np.array_equal(host(xs2).view(np.uint32), x[ref].view(np.uint32))
    assert bits_equal(y3, X.matvec_sym_unsorted(a_d, x_d)[0])
    X.device_status()
