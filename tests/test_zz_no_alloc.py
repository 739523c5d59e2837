"""The MLP call that allocates nothing and takes no scratch (svdq_gemm_swiglu_quant_noscratch), for
callers that cannot allocate device memory: a plug-in inside a framework that owns every device
allocation, or latency-bound code that cannot afford cudaMalloc's implicit synchronisation. Its
partial sums live in a fixed 8 MiB buffer in the library's device image.

Checked through the C ABI against the entry point that takes caller scratch
(svdq_gemm_swiglu_quant), on two calls in a row of different shapes (the second call runs over the
buffer contents the first left behind): the down layer's E2M1 codes, E4M3 scales and alpha
bit-identical, U' within 1e-4 of max|U'| (the bar the fused-chain tests use). A call too large for
the buffer is refused on the host before anything is enqueued.

This file sorts last so that a run stopping at its first failure has run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

from bit_diffusion_transformer_svdquant_b200 import _lib
from oracle import svdquant


def _rand(M, K, N, seed, outlier=50.0):
    rng = np.random.default_rng(seed)
    X = rng.standard_normal((M, K))
    X[:, rng.choice(K, max(1, K // 100), replace=False)] *= outlier
    X = svdquant.bf16_round(X)
    W = svdquant.bf16_round(rng.standard_normal((N, K)) / np.sqrt(K))
    b = svdquant.bf16_round(rng.standard_normal(N) * np.sqrt(0.02))
    return X, W, b


def _dev(a, dtype, dev):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(dtype).to(dev)


def _layer(X_cal, W, r, swiglu, dev):
    p = svdquant.prepare_layer(X_cal, W, r)
    return _lib.PackedWeight(_dev(p["R"], torch.float32, dev), _dev(p["L1s"], torch.bfloat16, dev) if r else None,
                             _dev(p["L2"], torch.bfloat16, dev) if r else None,
                             _dev(p["inv_lambda"], torch.float32, dev), swiglu=swiglu)


def _chain(M, K, N_up, N_dn, r_up, r_dn, seed, dev):
    """Gate/up layer quantized and ready, the down layer packed and calibrated on the unfused h."""
    X, W_up, b_up = _rand(M, K, N_up, seed)
    X2, W_dn, _ = _rand(M, N_up // 2, N_dn, seed + 1)
    w_up = _layer(X, W_up, r_up, True, dev)
    w_dn = _layer(X2, W_dn, r_dn, False, dev)
    Xd, bu = _dev(X, torch.bfloat16, dev), _dev(b_up, torch.bfloat16, dev)
    act_up = _lib.QuantizedAct(M, K, r_up, dev)
    _lib.quantize_act(Xd, w_up, _lib.calibrate_act(Xd, w_up), act_up)
    g_dn = _lib.calibrate_act(_lib.gemm(act_up, w_up, bu), w_dn)
    return {"M": M, "w_up": w_up, "w_dn": w_dn, "bu": bu, "act_up": act_up, "g_dn": g_dn}


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


@pytest.mark.gpu
def test_noscratch_matches_caller_scratch_twice_in_a_row(cuda_device):
    L = _lib.lib()
    stream = ctypes.c_void_p(torch.cuda.current_stream(cuda_device).cuda_stream)
    cases = [_chain(300, 512, 1024, 384, 16, 32, 5, cuda_device),      # 4 column tiles, next rank 32
             _chain(1100, 256, 2560, 256, 32, 16, 9, cuda_device)]     # 10 tiles, ragged rows, rank 16
    outs = []
    for c in cases:       # the no-scratch entry point, called twice in a row
        a = _lib.QuantizedAct(c["M"], c["w_dn"].K, c["w_dn"].r, cuda_device)
        rc = L.svdq_gemm_swiglu_quant_noscratch(ctypes.byref(c["act_up"].desc), ctypes.byref(c["w_up"].desc),
                                                _p(c["bu"]), ctypes.byref(c["w_dn"].desc), _p(c["g_dn"]),
                                                ctypes.byref(a.desc), None, stream)
        assert rc == 0, L.svdq_last_error()
        outs.append(a)
    refs = []
    for c in cases:       # the entry point with caller scratch
        a = _lib.QuantizedAct(c["M"], c["w_dn"].K, c["w_dn"].r, cuda_device)
        need = L.svdq_mlp_scratch_bytes(c["M"], c["w_dn"].r)
        scratch = torch.empty(need, dtype=torch.uint8, device=cuda_device)
        rc = L.svdq_gemm_swiglu_quant(ctypes.byref(c["act_up"].desc), ctypes.byref(c["w_up"].desc), _p(c["bu"]),
                                      ctypes.byref(c["w_dn"].desc), _p(c["g_dn"]), ctypes.byref(a.desc),
                                      _p(scratch), need, None, stream)
        assert rc == 0, L.svdq_last_error()
        refs.append((a, scratch))
    torch.cuda.synchronize(cuda_device)
    assert _lib.device_status() == 0
    for c, a, (ref, _) in zip(cases, outs, refs):
        M = c["M"]
        ca, sa = _lib.export_act(a)
        cr, sr = _lib.export_act(ref)
        assert torch.equal(sa, sr)
        assert torch.equal(ca, cr)
        assert float(a.alpha().item()) == float(ref.alpha().item())
        u = a.U()[:, :M].float().sum(0)
        u_ref = ref.U()[:, :M].float().sum(0)
        assert float((u - u_ref).abs().max()) <= 1e-4 * float(u_ref.abs().max())


def test_noscratch_refuses_calls_beyond_the_builtin_buffer():
    """At next-layer rank 32 the 8 MiB buffer holds M <= 8192 tokens; M = 8193 is refused with
    SVDQ_ERR_UNSUPPORTED on the host (descriptors bound over a fake address: nothing is enqueued)."""
    L = _lib.lib()
    base = ctypes.c_void_p(1 << 40)
    assert L.svdq_mlp_scratch_bytes(8192, 32) == 8 << 20
    w = _lib.SvdqWeight()
    w_next = _lib.SvdqWeight()
    w_next.r = 32
    act = _lib.SvdqAct()
    act_next = _lib.SvdqAct()
    assert L.svdq_act_bind(8193, 3072, 32, base, L.svdq_act_bytes(8193, 3072, 32), ctypes.byref(act)) == 0
    assert L.svdq_act_bind(8193, 12288, 32, base, L.svdq_act_bytes(8193, 12288, 32), ctypes.byref(act_next)) == 0
    rc = L.svdq_gemm_swiglu_quant_noscratch(ctypes.byref(act), ctypes.byref(w), None, ctypes.byref(w_next), base,
                                            ctypes.byref(act_next), None, None)
    assert rc == 2
    assert "built-in buffer" in L.svdq_last_error().decode()
    assert L.svdq_gemm_swiglu_quant_noscratch(None, ctypes.byref(w), None, ctypes.byref(w_next), base,
                                              ctypes.byref(act_next), None, None) == 1
