"""GPU parity: the CUDA path (through the C ABI) against the oracle on the same seeded inputs.

Bar: tensor scales, E2M1 codes and E4M3 scales bit-exact; fp32 outputs within
max|y - y_ref| <= 2e-3 * max|y_ref|; bf16 outputs bitwise equal to the bf16 rounding of the fp32
outputs; repeated runs bitwise identical.
"""
import numpy as np
import pytest
import torch

import bit_diffusion_transformer_svdquant_b200 as svdq
from bit_diffusion_transformer_svdquant_b200 import synth
from oracle import nvfp4, svdquant

from _parity import Case

pytestmark = pytest.mark.gpu


def _rand_layer(M, K, N, r, seed, bias=True, outlier=50.0):
    rng = np.random.default_rng(seed)
    X = rng.standard_normal((M, K))
    X[:, rng.choice(K, max(1, K // 100), replace=False)] *= outlier
    X = svdquant.bf16_round(X)
    W = svdquant.bf16_round(rng.standard_normal((N, K)) / np.sqrt(K))
    b = svdquant.bf16_round(rng.standard_normal(N) * np.sqrt(0.02)) if bias else None
    return X, W, b


def test_watchdog_selftest_returns_status(cuda_device):
    assert svdq.device_status(reset=True) == 0
    svdq.watchdog_selftest(2_000_000, cuda_device)       # 2 ms wait that nothing ends
    assert svdq.device_status(reset=True) == 4            # SVDQ_ERR_TIMEOUT, context still usable
    assert svdq.device_status(reset=True) == 0
    x = torch.ones(4, device=cuda_device)
    assert float(x.sum().item()) == 4.0


def test_codec_edges_through_kernel1(cuda_device):
    """Hand-built blocks that land exactly on E2M1 and E4M3 rounding ties, E4M3 subnormal and zero
    scales, saturation and signed zeros, pushed through the activation kernel with lambda = 1 and a
    static g_x = 1 (so that block values reach the codecs unscaled; row 2 exceeds the calibrated
    range and saturates)."""
    K, M = 256, 32
    rng = np.random.default_rng(11)
    X = svdquant.bf16_round(rng.standard_normal((M, K)))
    X[1, 0:16] = [6, 0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5, -0.25, -0.75, -1.25, -1.75, -2.5, -3.5, -5, -0.1015625]
    X[1, 16:32] = [6.375] + [1.0] * 15                   # amax/6 = 1.0625: E4M3 tie -> 1.0
    X[1, 32:48] = [7.125] + [-0.5] * 15                  # amax/6 = 1.1875: tie -> 1.25
    X[1, 48:64] = [6 * 2.0 ** -10] + [1e-4] * 15         # amax/6 = 2^-10: tie -> 0 -> zero block
    X[1, 64:80] = [6 * 1.5 * 2.0 ** -9] + [0.001] * 15   # tie between 1 and 2 subnormal steps -> 2
    X[1, 80:96] = 0.0
    X[1, 96:112] = -0.0
    X[2, :] = svdquant.bf16_round(rng.standard_normal(K) * 1e4)   # saturating scales and codes
    X = svdquant.bf16_round(X)
    W = svdquant.bf16_round(rng.standard_normal((128, K)) / 16)
    prep = {"inv_lambda": np.ones(K), "lam_prime": np.ones(K), "L1s": np.zeros((K, 0)), "L2": np.zeros((0, 128)),
            "R": nvfp4.f32(W), "r": 0}
    c = Case(X, W, None, 0, False, cuda_device, prep=prep, g_x=1.0)
    c.check_scales()
    c.check_act_codes()
    c.check_weight_codes()
    c.check_outputs()


SMALL_CASES = [
    # M, K, N, r, bias, swiglu     (tile width: 384 without SwiGLU where 768 divides N, else 256
    # where it divides N, else 192, else 128)
    (300, 768, 384, 32, True, False),   # ragged M (odd number of 128-row blocks), two 192-wide tiles
    (1, 256, 128, 0, False, False),     # one row, no low-rank branch, 128-wide tile
    (200, 512, 768, 64, True, True),    # SwiGLU with bias, r = 64, three 256-wide tiles
    (130, 1024, 256, 16, False, True),  # SwiGLU, no bias, one 256-wide tile
    (513, 256, 192, 32, False, False),  # a ragged fifth m-tile, K = one k-step
    (1000, 2048, 1152, 32, True, False),
    (257, 512, 640, 32, True, True),    # SwiGLU on 128-wide tiles (double-buffered accumulators)
    (600, 768, 1024, 32, True, False),  # four 256-wide tiles, ragged M
    (170, 512, 384, 32, True, True),    # SwiGLU on 192-wide tiles (2 + 1 output chunks per quadrant)
    (300, 768, 768, 32, True, False),   # 384-wide tiles (two MMAs per K chunk), ragged M
    (1, 256, 768, 0, False, False),     # 384-wide, one row, no low-rank branch
    (130, 1024, 768, 16, False, False), # 384-wide, r = 16 (32-byte low-rank rows)
    (513, 256, 1536, 64, True, False),  # 384-wide, r = 64 (two low-rank slots), a ragged fifth m-tile
]


@pytest.mark.parametrize("M,K,N,r,bias,swiglu", SMALL_CASES)
def test_small_shapes(cuda_device, M, K, N, r, bias, swiglu):
    X, W, b = _rand_layer(M, K, N, r, seed=M * 7 + N, bias=bias)
    c = Case(X, W, b, r, swiglu, cuda_device)
    assert c.w.n_tile == (384 if not swiglu and N % 768 == 0 else 256 if N % 256 == 0 else 192 if N % 192 == 0
                          else 128)
    c.check_scales()
    c.check_weight_codes()
    c.check_act_codes()
    c.check_outputs()


def test_tiny_workload(cuda_device):
    spec = synth.WORKLOADS["tiny"].layers[0]
    d = synth.make_linear_inputs(spec)
    c = Case(synth.bf16_values(d["X"]), synth.bf16_values(d["W"]), None, spec.r, False, cuda_device)
    c.check_scales()
    c.check_weight_codes()
    c.check_act_codes()
    c.check_outputs()


def test_repeatable(cuda_device):
    X, W, b = _rand_layer(384, 512, 384, 32, seed=5)
    c = Case(X, W, b, 32, False, cuda_device)
    y1 = c.run_gemm(torch.float32).clone()
    u1 = c.act.U().clone()
    svdq.quantize_act(c.Xd, c.w, c.g_x, c.act)
    y2 = c.run_gemm(torch.float32)
    assert torch.equal(u1, c.act.U())
    assert torch.equal(y1, y2)


def _full_layers():
    out = []
    for wl in synth.WORKLOADS.values():
        if wl.name == "tiny":
            continue
        for spec in wl.layers:
            out.append(pytest.param(spec, id=spec.name))
    return out


@pytest.mark.slow
@pytest.mark.parametrize("spec", _full_layers())
def test_full_size_workload(cuda_device, spec):
    """Every layer of every workload at its full size: all codes and scales bit-exact, outputs on a
    few thousand sampled positions (plus tile corners and the last row) within tolerance."""
    d = synth.make_linear_inputs(spec)
    X, W = synth.bf16_values(d["X"]), synth.bf16_values(d["W"])
    b = synth.bf16_values(d["bias"]) if spec.bias else None
    c = Case(X, W, b, spec.r, spec.swiglu, cuda_device)
    c.check_scales()
    c.check_weight_codes()
    c.check_act_codes()
    c.check_outputs(samples=3000)


@pytest.mark.parametrize("N", [512, 768])  # 256- and 384-wide GEMM tiles
def test_cuda_graph_replay(cuda_device, N):
    """Both kernels captured in a CUDA graph and replayed give the eager result bit for bit (the
    library enqueues everything on the caller's stream and allocates nothing per call), in bf16 and
    fp32 output modes; the replayed activation codes and scales equal the oracle's, and the replayed
    fp32 output is within 2e-3 of max|y_ref| of the oracle's layer."""
    X, W, b = _rand_layer(300, 768, N, 32, seed=11, bias=True)
    c = Case(X, W, b, 32, False, cuda_device)
    for dt in (torch.bfloat16, torch.float32):
        y_eager = c.run_gemm(dt).clone()
        Y = torch.empty_like(y_eager)
        side = torch.cuda.Stream(cuda_device)
        side.wait_stream(torch.cuda.current_stream(cuda_device))
        with torch.cuda.stream(side):
            svdq.quantize_act(c.Xd, c.w, c.g_x, c.act)
            svdq.gemm(c.act, c.w, c.bias_d, out=Y, out_dtype=dt)
        torch.cuda.current_stream(cuda_device).wait_stream(side)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            svdq.quantize_act(c.Xd, c.w, c.g_x, c.act)
            svdq.gemm(c.act, c.w, c.bias_d, out=Y, out_dtype=dt)
        Y.zero_()
        c.act.buf.zero_()        # the replay must rewrite codes, scales, U and alpha itself
        g.replay()
        torch.cuda.synchronize(cuda_device)
        assert svdq.device_status() == 0
        assert torch.equal(Y, y_eager)
        c.check_act_codes()
        if dt == torch.float32:
            y = Y.cpu().numpy().astype(np.float64)
            ref = c.y_ref_full()
            assert np.max(np.abs(y - ref)) <= 2e-3 * np.max(np.abs(ref))
        del g


@pytest.mark.parametrize("N", [512, 768])  # 256- and 384-wide GEMM tiles
def test_lora_on_the_branch(cuda_device, N):
    """A rank-32 LoRA adapter concatenated onto the rank-32 branch (r = 64 through the same
    kernels) matches the oracle's base layer + X A B."""
    X, W, b = _rand_layer(300, 768, N, 32, seed=13, bias=True)
    rng = np.random.default_rng(17)
    A = svdquant.bf16_round(rng.standard_normal((768, 32)) / np.sqrt(768))
    B = svdquant.bf16_round(rng.standard_normal((32, N)) * 0.05)
    prep = svdquant.add_lora(svdquant.prepare_layer(X, W, 32), A, B)
    c = Case(X, W, b, 64, False, cuda_device, prep=prep)
    c.check_scales()
    c.check_weight_codes()
    c.check_act_codes()
    c.check_outputs()


def test_dynamic_activation_scale(cuda_device):
    """linear() without g_x computes the scale from the call's own X (the amax pass) and gives
    exactly the result of the statically calibrated path on the same X; the scale is the oracle's."""
    X, W, b = _rand_layer(260, 512, 384, 16, seed=21, bias=True)
    c = Case(X, W, b, 16, False, cuda_device)
    y_static = svdq.linear(c.Xd, c.w, c.g_x, c.bias_d)
    y_dynamic = svdq.linear(c.Xd, c.w, None, c.bias_d)
    torch.cuda.synchronize(cuda_device)
    assert torch.equal(y_static, y_dynamic)
    assert float(svdq.calibrate_act(c.Xd, c.w).item()) == c.g_x_ref


@pytest.mark.parametrize("M,K,N,r,swiglu", [(130, 256, 384, 16, False), (200, 512, 512, 32, True),
                                            (130, 256, 768, 16, False)])
def test_outputs_stay_inside_y(cuda_device, M, K, N, r, swiglu):
    """Canaries: Y is the first M rows of a larger buffer filled with a marker value; after the GEMM
    the rows past M still hold the marker (the output TMA stores clip at row M, although the tile
    computes M_pad rows), and Y equals the output of a call into a fresh tensor."""
    X, W, _ = _rand_layer(M, K, N, r, seed=M + N, bias=False)
    c = Case(X, W, None, r, swiglu, cuda_device)
    n_out = N // 2 if swiglu else N
    marker = -7680.0  # exact in bf16 and fp32
    for dt in (torch.bfloat16, torch.float32):
        big = torch.full((M + 64, n_out), marker, dtype=dt, device=cuda_device)
        y = svdq.gemm(c.act, c.w, None, out=big[:M], out_dtype=dt)
        fresh = svdq.gemm(c.act, c.w, None, out_dtype=dt)
        torch.cuda.synchronize(cuda_device)
        assert svdq.device_status() == 0
        assert torch.all(big[M:] == marker)
        assert torch.equal(y, fresh)


MULTI_TILE = [
    # more tiles than resident CTA pairs on 384-, 192- and 128-wide tiles (the full-size workloads
    # use 384- and 256-wide ones): the 128-wide kernel's double-buffered accumulators and the
    # barrier phases carried from tile to tile.      pair tiles = ceil(M / 256) x N / n_tile
    (2048, 512, 4736, 32, True, False),   # 128-wide: 8 x 37 = 296 tiles
    (1280, 256, 4736, 16, False, True),   # 128-wide SwiGLU: 5 x 37 = 185 tiles
    (1536, 512, 5760, 32, True, False),   # 192-wide: 6 x 30 = 180 tiles
    (1100, 256, 5760, 64, True, True),    # 192-wide SwiGLU, r = 64, ragged last row block: 5 x 30
    (2048, 512, 9216, 32, True, False),   # 384-wide: 8 x 24 = 192 tiles
    (1100, 256, 6912, 16, False, False),  # 384-wide, ragged last row block: 5 x 18 = 90 tiles
]


@pytest.mark.parametrize("M,K,N,r,bias,swiglu", MULTI_TILE)
def test_multi_tile_per_pair(cuda_device, M, K, N, r, bias, swiglu):
    X, W, b = _rand_layer(M, K, N, r, seed=3 * M + N, bias=bias)
    c = Case(X, W, b, r, swiglu, cuda_device)
    c.check_scales()
    c.check_weight_codes()
    c.check_act_codes()
    c.check_outputs()


@pytest.mark.parametrize("M", [127, 128, 129, 255, 256])
def test_row_block_boundaries(cuda_device, M):
    """M on either side of a 128-row block and of a 256-row pair: a partial block, an exact pair, a
    pair whose odd CTA has no rows, and one block plus a row."""
    X, W, b = _rand_layer(M, 256, 256, 16, seed=1000 + M, bias=True)
    c = Case(X, W, b, 16, False, cuda_device)
    c.check_scales()
    c.check_act_codes()
    c.check_outputs()


_DESC_PTRS = ("codes", "scales", "g_w", "inv_lambda", "L1s_t", "L2_t")


def test_packed_weight_checkpoint_round_trip(cuda_device):
    """A packed weight saved to the host (state_dict) and re-bound at another device address
    (from_state, svdq_weight_bind) gives the GEMM bit-identical outputs; SwiGLU packing included.
    The original blob is overwritten before the restored weight runs, so a bind that kept the old
    TMA descriptors (or pointers) would read garbage and fail."""
    for swiglu in (False, True):
        X, W, b = _rand_layer(300, 512, 768, 32, seed=77 + swiglu, bias=True)
        c = Case(X, W, b, 32, swiglu, cuda_device)
        y0 = c.run_gemm(torch.float32)
        restored = svdq.PackedWeight.from_state(c.w.state_dict(), cuda_device)
        assert restored.buf.data_ptr() != c.w.buf.data_ptr()
        lo, hi = restored.buf.data_ptr(), restored.buf.data_ptr() + restored.buf.numel()
        for f in _DESC_PTRS:
            assert lo <= getattr(restored.desc, f) < hi, f
        g = torch.Generator(device=cuda_device).manual_seed(5)
        c.w.buf.copy_(torch.randint(0, 256, c.w.buf.shape, generator=g, device=cuda_device, dtype=torch.int32)
                      .to(torch.uint8))
        y1 = svdq.gemm(c.act, restored, c.bias_d, out_dtype=torch.float32)
        torch.cuda.synchronize(cuda_device)
        assert svdq.device_status() == 0
        assert torch.equal(y0, y1)


def test_weight_bind_offsets_match_pack(cuda_device):
    """A bind of an (uninitialised) blob puts every descriptor pointer at the offset a pack into a
    buffer of the same shape produces, relative to each buffer's start."""
    X, W, b = _rand_layer(256, 512, 768, 32, seed=79, bias=False)
    c = Case(X, W, None, 32, False, cuda_device)
    blob = torch.empty_like(c.w.buf)
    lib = svdq._lib.lib()
    d = svdq._lib.SvdqWeight()
    import ctypes
    assert lib.svdq_weight_bind(c.w.N, c.w.K, c.w.r, 0, c.w.n_tile, ctypes.c_void_p(blob.data_ptr()),
                                blob.numel(), ctypes.byref(d)) == 0
    for f in _DESC_PTRS:
        assert getattr(d, f) - blob.data_ptr() == getattr(c.w.desc, f) - c.w.buf.data_ptr(), f
    assert (d.N, d.K, d.r, d.n_tile, d.swiglu_interleaved) == (c.w.N, c.w.K, c.w.r, c.w.n_tile, 0)


@pytest.mark.parametrize("r", [16, 32, 64])
@pytest.mark.parametrize("cluster", ["1", "2", "3", "4"])
def test_kernel1_cluster_sizes(cuda_device, monkeypatch, cluster, r):
    """Kernel 1 with K split over thread-block clusters of 1 to 4 CTAs (SVDQ_K1_CLUSTER), at every
    branch rank: the leader's sum of its peers' partial U (16-byte loads up to r = 32, 4-byte loads
    at r = 64) must keep codes and scales bit-exact and the outputs within 2e-3 of the oracle, and
    U must not depend on the split (the sums run in rank order; rounding aside, the same values)."""
    X, W, b = _rand_layer(300, 768, 512, r, seed=77 + r, bias=True)
    monkeypatch.setenv("SVDQ_K1_CLUSTER", cluster)
    c = Case(X, W, b, r, False, cuda_device)
    c.check_scales()
    c.check_act_codes()
    c.check_outputs()
    u_split = c.act.U().float().clone()
    monkeypatch.setenv("SVDQ_K1_CLUSTER", "1")
    svdq.quantize_act(c.Xd, c.w, c.g_x, c.act)
    torch.cuda.synchronize(cuda_device)
    assert svdq.device_status() == 0
    u_one = c.act.U().float()
    # hi + lo of U: fp32 partial sums in another order differ by rounding only
    tot_split, tot_one = u_split[0] + u_split[1], u_one[0] + u_one[1]
    assert float((tot_split - tot_one).abs().max()) <= 1e-4 * float(tot_one.abs().max()) + 1e-30
