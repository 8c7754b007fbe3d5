"""Concurrency and graph capture of the C-ABI calls:
* GEMMs launched concurrently on two streams (each launch takes its own
  pacing-counter slot) give exactly the results of the same calls run one
  after the other -- every output element is computed by one CTA in a fixed
  order, so the kernels are deterministic;
* the quantizer and the GEMM calls captured into a CUDA graph (after the
  device's one-time set-up) replay to the eager results on new inputs;
* the same for the one-call quantizing Linear and the multi-Linear GEMMs."""
import pytest
import torch

from int8_w8a8_quantized_b200 import _capi, workloads
from tests import _gpu

pytestmark = pytest.mark.gpu


def _codes(g, shape):
    mag = torch.randint(0, 0x70, shape, generator=g, dtype=torch.int32)
    return (mag | (torch.randint(0, 2, shape, generator=g, dtype=torch.int32) << 7)).to(torch.uint8).cuda()


def _gemm(lib, A, sa, W, sw, b, y, stream):
    M, K = A.shape
    N = W.shape[0]
    st = lib.tfq_scaled_fp8_linear(A.data_ptr(), sa.data_ptr(), W.data_ptr(), sw.data_ptr(),
                                   None if b is None else b.data_ptr(), M, N, K, y.data_ptr(),
                                   int(stream.cuda_stream))
    assert st == _capi.TFQ_OK, _capi.last_error_message()


def test_concurrent_streams_match_serial():
    lib = _gpu.lib()
    g = torch.Generator().manual_seed(11)
    cases = []
    for (M, N, K) in [(3000, 3072, 1024), (2048, 1032, 2048), (700, 520, 512)]:
        A, W = _codes(g, (M, K)), _codes(g, (N, K))
        sa = (torch.rand(M, generator=g) * 1e-2).cuda()
        sw = (torch.rand(N, generator=g) * 1e-2).cuda()
        b = torch.randn(N, generator=g).to(torch.bfloat16).cuda()
        cases.append((A, sa, W, sw, b))
    main = torch.cuda.current_stream()
    serial = []
    for c in cases:
        y = torch.empty((c[0].shape[0], c[2].shape[0]), dtype=torch.bfloat16, device="cuda")
        _gemm(lib, *c, y, main)
        serial.append(y)
    torch.cuda.synchronize()
    streams = [torch.cuda.Stream() for _ in cases]
    conc = [torch.empty_like(y) for y in serial]
    for _ in range(3):
        for c, y, s in zip(cases, conc, streams):
            s.wait_stream(main)
            _gemm(lib, *c, y, s)
        for s in streams:
            main.wait_stream(s)
        torch.cuda.synchronize()
        for a, b in zip(serial, conc):
            assert torch.equal(a, b)
    _gpu.check_device_error()


def test_cuda_graph_capture_and_replay():
    lib = _gpu.lib()
    M, K, N = 1500, 1024, 776
    x = workloads.activations(M, K, seed=5, outlier_cols=4, outlier_mult=20.0, device="cuda")
    w = workloads.weights(N, K, seed=6, std=0.02, device="cuda")
    b = workloads.bias(N, seed=7, device="cuda")
    Wq, sw = _gpu.quant_weight(w, _capi.TFQ_DTYPE_FP8_E4M3, 448.0)
    A = torch.empty((M, K), dtype=torch.uint8, device="cuda")
    sa = torch.empty(M, device="cuda")
    y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")

    def linear(stream):
        sh = int(stream.cuda_stream)
        assert lib.tfq_quant_act_fp8_per_token(x.data_ptr(), M, K, 448.0, A.data_ptr(), sa.data_ptr(), sh) == 0
        assert lib.tfq_scaled_fp8_linear(A.data_ptr(), sa.data_ptr(), Wq.data_ptr(), sw.data_ptr(), b.data_ptr(),
                                         M, N, K, y.data_ptr(), sh) == 0

    linear(torch.cuda.current_stream())          # one-time set-up happens outside the capture
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        with torch.cuda.graph(graph, stream=side):
            linear(side)
    torch.cuda.current_stream().wait_stream(side)
    for seed in (8, 9):
        x.copy_(workloads.activations(M, K, seed=seed, nu=4, device="cuda"))
        graph.replay()
        torch.cuda.synchronize()
        y_graph = y.clone()
        linear(torch.cuda.current_stream())
        torch.cuda.synchronize()
        assert torch.equal(y_graph, y)
    del graph
    _gpu.check_device_error()


def test_mxfp8_and_int8_concurrent_streams_match_serial():
    """The MXFP8 and INT8 paths on two streams at once give the results of the
    same calls run one after the other."""
    from int8_w8a8_quantized_b200 import tfq_mxfp8_linear, tfq_quant_mxfp8, tfq_quant_weight_per_channel
    from int8_w8a8_quantized_b200 import tfq_quant_act_int8_per_token, tfq_scaled_int8_linear
    _gpu.lib()
    x = workloads.activations(2048, 1024, seed=21, device="cuda")
    w = workloads.weights(2560, 1024, seed=22, std=0.02, device="cuda")
    b = workloads.bias(2560, seed=23, device="cuda")
    Wm, sfw = tfq_quant_mxfp8(w)
    Wi, swi = tfq_quant_weight_per_channel(w, "int8")
    Am, sfa = tfq_quant_mxfp8(x)
    Ai, sai = tfq_quant_act_int8_per_token(x)
    torch.cuda.synchronize()
    ref_m = tfq_mxfp8_linear(Am, sfa, Wm, sfw, b)
    ref_i = tfq_scaled_int8_linear(Ai, sai, Wi, swi, b)
    torch.cuda.synchronize()
    s1, s2 = torch.cuda.Stream(), torch.cuda.Stream()
    for _ in range(3):
        s1.wait_stream(torch.cuda.current_stream())
        s2.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s1):
            y_m = tfq_mxfp8_linear(Am, sfa, Wm, sfw, b, stream=s1)
        with torch.cuda.stream(s2):
            y_i = tfq_scaled_int8_linear(Ai, sai, Wi, swi, b, stream=s2)
        torch.cuda.current_stream().wait_stream(s1)
        torch.cuda.current_stream().wait_stream(s2)
        torch.cuda.synchronize()
        assert torch.equal(y_m, ref_m) and torch.equal(y_i, ref_i)
    _gpu.check_device_error()


def test_pacing_slots_reused_eager_and_in_a_graph():
    """A pair-kernel GEMM launched 70 times in a row (more launches than
    pacing-counter slots, so slots are reused; each launch leaves its slot at
    zero for the next) and replayed 5 times from a CUDA graph (the same slot
    every replay): every result equals the first, no bounded wait runs out."""
    lib = _gpu.lib()
    g = torch.Generator().manual_seed(5)
    M, N, K = 2048, 2048, 512  # 64 pair tiles on 64 clusters
    A, W = _codes(g, (M, K)), _codes(g, (N, K))
    sa = (torch.rand(M, generator=g) * 1e-2).cuda()
    sw = (torch.rand(N, generator=g) * 1e-2).cuda()
    b = torch.randn(N, generator=g).to(torch.bfloat16).cuda()
    main = torch.cuda.current_stream()
    ref = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    _gemm(lib, A, sa, W, sw, b, ref, main)
    y = torch.empty_like(ref)
    for _ in range(70):
        y.fill_(0)
        _gemm(lib, A, sa, W, sw, b, y, main)
    torch.cuda.synchronize()
    assert torch.equal(y, ref)
    _gpu.check_device_error()
    s = torch.cuda.Stream()
    yg = torch.zeros_like(ref)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        _gemm(lib, A, sa, W, sw, b, yg, s)  # warm up on the capture stream
        torch.cuda.synchronize()
        with torch.cuda.graph(graph, stream=s):
            _gemm(lib, A, sa, W, sw, b, yg, s)
    for _ in range(5):
        yg.fill_(0)
        graph.replay()
        torch.cuda.synchronize()
        assert torch.equal(yg, ref)
    _gpu.check_device_error()


def test_one_call_quant_linear_graph_and_concurrent_streams():
    """The one-call quantization + GEMM (its workspace clear and its kernel)
    captured into a CUDA graph replays to the eager result on new inputs; two
    calls with workspaces of their own run concurrently on two streams and give
    the results of the same calls run one after the other."""
    lib = _gpu.lib()
    cases = []
    for i, (M, K, N) in enumerate([(2600, 1024, 1032), (1800, 3072, 776)]):
        x = workloads.activations(M, K, seed=30 + i, outlier_cols=8, outlier_mult=20.0, device="cuda")
        w = workloads.weights(N, K, seed=40 + i, std=0.02, device="cuda")
        b = workloads.bias(N, seed=50 + i, device="cuda")
        Wq, sw = _gpu.quant_weight(w, _capi.TFQ_DTYPE_FP8_E4M3, 448.0)
        A = torch.empty((M, K), dtype=torch.uint8, device="cuda")
        sa = torch.empty(M, device="cuda")
        y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
        ws = torch.empty(lib.tfq_quant_scaled_fp8_linear_workspace_bytes(M), dtype=torch.uint8, device="cuda")
        cases.append((x, Wq, sw, b, A, sa, y, ws))

    def call(c, stream):
        x, Wq, sw, b, A, sa, y, ws = c
        M, K = x.shape
        st = lib.tfq_quant_scaled_fp8_linear(x.data_ptr(), M, K, 448.0, Wq.data_ptr(), sw.data_ptr(), b.data_ptr(),
                                             Wq.shape[0], A.data_ptr(), sa.data_ptr(), y.data_ptr(), ws.data_ptr(),
                                             int(stream.cuda_stream))
        assert st == _capi.TFQ_OK, _capi.last_error_message()

    main = torch.cuda.current_stream()
    for c in cases:
        call(c, main)
    torch.cuda.synchronize()
    serial = [c[6].clone() for c in cases]
    # concurrent streams, a workspace each
    streams = [torch.cuda.Stream() for _ in cases]
    for _ in range(3):
        for c in cases:
            c[6].zero_()
        for c, s in zip(cases, streams):
            s.wait_stream(main)
            call(c, s)
        for s in streams:
            main.wait_stream(s)
        torch.cuda.synchronize()
        for c, ref in zip(cases, serial):
            assert torch.equal(c[6], ref)
    # graph capture of the first call, replayed on new inputs
    c = cases[0]
    graph = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream()
    side.wait_stream(main)
    with torch.cuda.stream(side):
        with torch.cuda.graph(graph, stream=side):
            call(c, side)
    main.wait_stream(side)
    M, K = c[0].shape
    for seed in (60, 61):
        c[0].copy_(workloads.activations(M, K, seed=seed, nu=4, device="cuda"))
        graph.replay()
        torch.cuda.synchronize()
        y_graph = c[6].clone()
        call(c, main)
        torch.cuda.synchronize()
        assert torch.equal(y_graph, c[6])
    del graph
    _gpu.check_device_error()


def test_multi_linear_graph_and_concurrent_streams():
    """Q/K/V-like multi-Linear launches (FP8 and INT8) on two streams at once,
    and one captured into a CUDA graph and replayed on new codes, give the
    results of the same calls run eagerly one after the other."""
    lib = _gpu.lib()
    g = torch.Generator().manual_seed(23)
    M, K, Ns = 2100, 1024, (1032, 520, 776)
    arr = _capi.pointer_array
    import ctypes

    def operands(int8):
        if int8:
            A = torch.randint(-128, 128, (M, K), generator=g, dtype=torch.int8).cuda()
            Ws = [torch.randint(-128, 128, (N, K), generator=g, dtype=torch.int8).cuda() for N in Ns]
        else:
            A, Ws = _codes(g, (M, K)), [_codes(g, (N, K)) for N in Ns]
        sa = (torch.rand(M, generator=g) * 1e-3).cuda()
        sws = [(torch.rand(N, generator=g) * 1e-3).cuda() for N in Ns]
        bs = [torch.randn(N, generator=g).to(torch.bfloat16).cuda() for N in Ns]
        ys = [torch.empty((M, N), dtype=torch.bfloat16, device="cuda") for N in Ns]
        return A, sa, Ws, sws, bs, ys

    def call(entry, ops, stream):
        A, sa, Ws, sws, bs, ys = ops
        st = getattr(lib, entry)(A.data_ptr(), sa.data_ptr(), M, K, len(Ns), arr([w.data_ptr() for w in Ws]),
                                 arr([s.data_ptr() for s in sws]), arr([b.data_ptr() for b in bs]),
                                 (ctypes.c_int64 * len(Ns))(*Ns), arr([y.data_ptr() for y in ys]),
                                 int(stream.cuda_stream))
        assert st == _capi.TFQ_OK, _capi.last_error_message()

    cases = [("tfq_scaled_fp8_linear_multi", operands(False)), ("tfq_scaled_int8_linear_multi", operands(True))]
    main = torch.cuda.current_stream()
    for entry, ops in cases:
        call(entry, ops, main)
    torch.cuda.synchronize()
    serial = [[y.clone() for y in ops[5]] for _, ops in cases]
    streams = [torch.cuda.Stream() for _ in cases]
    for _ in range(3):
        for (_, ops) in cases:
            for y in ops[5]:
                y.zero_()
        for (entry, ops), s in zip(cases, streams):
            s.wait_stream(main)
            call(entry, ops, s)
        for s in streams:
            main.wait_stream(s)
        torch.cuda.synchronize()
        for (_, ops), ref in zip(cases, serial):
            for y, r in zip(ops[5], ref):
                assert torch.equal(y, r)
    entry, ops = cases[0]
    graph = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream()
    side.wait_stream(main)
    with torch.cuda.stream(side):
        with torch.cuda.graph(graph, stream=side):
            call(entry, ops, side)
    main.wait_stream(side)
    for _ in range(2):
        ops[0].copy_(_codes(g, (M, K)))
        graph.replay()
        torch.cuda.synchronize()
        y_graph = [y.clone() for y in ops[5]]
        call(entry, ops, main)
        torch.cuda.synchronize()
        for a, b in zip(y_graph, ops[5]):
            assert torch.equal(a, b)
    del graph
    _gpu.check_device_error()
