"""The C-ABI library builds, loads without a GPU, exports every entry point include/svdq.h declares,
and its host-side logic (size queries, layouts, argument checks) behaves; no compute call is made."""
import ctypes
import os

import pytest

from bit_diffusion_transformer_svdquant_b200 import _lib, build


@pytest.fixture(scope="module")
def L():
    build.build()
    return _lib.lib()


def test_exports_every_declared_symbol(L):
    names = _lib.header_functions()
    assert len(names) >= 15
    raw = ctypes.CDLL(_lib.LIB_PATH)
    for n in names:
        assert hasattr(raw, n), n
    assert L.svdq_abi_version() == 1


def test_status_strings(L):
    for s in range(5):
        assert L.svdq_status_str(s)


def test_size_queries(L):
    # QKV 3072 -> 9216, r = 32 at n_tile 256: codes + 2-atom scales + g_w + inv_lambda + L1s^T + L2^T
    nb = L.svdq_weight_bytes(9216, 3072, 32)
    assert nb >= 9216 * 1536 + 9216 // 256 * 48 * 2 * 512 + 3072 * 4 + 32 * 3072 * 2 + 9216 * 32 * 2
    assert L.svdq_weight_bytes(9216, 3000, 32) == 0          # K % 256
    assert L.svdq_weight_bytes(9216, 3072, 24) == 0          # r not in {0,16,32,64}
    assert L.svdq_weight_bytes(100, 3072, 32) == 0           # N not a multiple of 128 or 192
    na = L.svdq_act_bytes(16896, 3072, 32)
    assert na >= 16896 * 1536 + 132 * 48 * 512 + 2 * 16896 * 32 * 2
    assert L.svdq_act_bytes(0, 3072, 32) == 0


def test_act_bind_layout(L):
    act = _lib.SvdqAct()
    base = 1 << 40
    M, K, r = 300, 512, 16
    nb = L.svdq_act_bytes(M, K, r)
    assert L.svdq_act_bind(M, K, r, ctypes.c_void_p(base), nb, ctypes.byref(act)) == 0
    assert act.M_pad == 384 and act.codes == base
    assert act.scales - act.codes >= 384 * 256 and act.scales % 256 == 0
    assert act.U - act.scales >= 3 * 8 * 512 and act.alpha - act.U >= 2 * 384 * 16 * 2
    assert L.svdq_act_bind(M, K, r, ctypes.c_void_p(base), nb - 1, ctypes.byref(act)) == 1
    assert L.svdq_act_bind(M, K, r, ctypes.c_void_p(base + 16), nb, ctypes.byref(act)) == 2


def test_argument_checks_before_any_cuda_call(L):
    w = _lib.SvdqWeight()
    p = ctypes.c_void_p(1 << 40)
    assert L.svdq_pack_weight(None, p, p, p, 512, 512, 16, 0, p, 1 << 30, ctypes.byref(w), None) == 1
    assert L.svdq_pack_weight(p, p, p, p, 500, 512, 16, 0, p, 1 << 30, ctypes.byref(w), None) == 2
    assert L.svdq_pack_weight(p, None, None, p, 512, 512, 16, 0, p, 1 << 30, ctypes.byref(w), None) == 1
    assert L.svdq_set_wait_limit_ns(10) == 1
    assert b"wait limit" in L.svdq_last_error()


def _fake_pair(L):
    """A weight and an act descriptor laid out as the pack / bind calls would, over fake addresses."""
    base = 1 << 40
    w = _lib.SvdqWeight(N=512, K=512, r=16, swiglu_interleaved=0, n_tile=256)
    for i, f in enumerate(("codes", "scales", "g_w", "inv_lambda", "L1s_t", "L2_t")):
        setattr(w, f, base + (i << 20))
    act = _lib.SvdqAct()
    assert L.svdq_act_bind(300, 512, 16, ctypes.c_void_p(base + (64 << 20)), 1 << 30, ctypes.byref(act)) == 0
    return w, act


@pytest.mark.parametrize("field,value", [("n_tile", 100), ("n_tile", 0), ("n_tile", 384), ("N", 640), ("K", 500),
                                         ("r", 24),
                                         ("codes", None), ("L2_t", None), ("M_pad", 256), ("M", 0),
                                         ("alpha", None), ("U", None)])
def test_descriptor_checks_before_any_cuda_call(L, field, value):
    """A hand-filled descriptor that no pack / bind call makes is rejected on the host (status 1)."""
    w, act = _fake_pair(L)
    p = ctypes.c_void_p(1 << 41)
    tgt = act if field in ("M_pad", "M", "alpha", "U") else w
    if field == "K":
        act.K = value
    setattr(tgt, field, value)
    assert L.svdq_gemm(ctypes.byref(act), ctypes.byref(w), None, 0, p, 0, None) == 1, L.svdq_last_error()
    assert L.svdq_quantize_act(p, ctypes.byref(w), p, ctypes.byref(act), None) == 1, L.svdq_last_error()
    if tgt is w:
        assert L.svdq_export_weight(ctypes.byref(w), p, p, None) == 1
        assert L.svdq_calibrate_act(p, 300, ctypes.byref(w), p, None) == 1
    else:
        assert L.svdq_export_act(ctypes.byref(act), p, p, None) == 1
    assert b"descriptor" in L.svdq_last_error()


def test_no_gpu_fails_loudly(L):
    """Valid arguments on a machine without a usable GPU: a CUDA error status, not a fallback."""
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    w = _lib.SvdqWeight()
    p = ctypes.c_void_p(1 << 40)
    st = L.svdq_pack_weight(p, p, p, p, 512, 512, 16, 0, p, 1 << 30, ctypes.byref(w), None)
    assert st == 3, (st, L.svdq_last_error())
    # well-formed descriptors get past the host checks and stop at the device query
    w, act = _fake_pair(L)
    st = L.svdq_gemm(ctypes.byref(act), ctypes.byref(w), None, 0, p, 0, None)
    assert st == 3, (st, L.svdq_last_error())


def _rank_main(rank, world, port, q):
    import os
    import torch
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    torch.distributed.init_process_group("gloo", rank=rank, world_size=world)
    import bench
    got = bench.max_over_ranks(1.5 + rank, torch.device("cpu"))
    torch.distributed.barrier()
    torch.distributed.destroy_process_group()
    q.put((rank, got))


def test_bench_max_over_ranks_gloo():
    """The N>1 bench path (replicas): the reported time is the slowest rank's, on a 2-rank gloo group."""
    import multiprocessing as mp
    import socket
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
    assert res == {0: 2.5, 1: 2.5}


def _weight_bytes_for_tile(N, K, r, n_tile):
    """Bytes of a weight blob laid out for a given tile width (each part 256-byte aligned)."""
    def up(x):
        return (x + 255) // 256 * 256
    atoms = (n_tile + 127) // 128
    parts = [N * K // 2, N // n_tile * (K // 64) * atoms * 512, 4, K * 4]
    if r:
        parts += [r * K * 2, N * r * 2]
    return sum(up(p) for p in parts)


@pytest.mark.parametrize("N,tile", [(512, 256), (9216, 256), (384, 192), (1152, 192), (640, 128), (128, 128)])
def test_tile_width_choice(L, N, tile):
    """256 where it divides N, else 192, else 128: visible in the scale-atom count of the blob. (Where
    768 divides N a weight without SwiGLU is packed 384 wide, whose blob has the size of the 256-wide
    one, so the size query need not know whether the weight is SwiGLU.)"""
    K, r = 512, 32
    got = L.svdq_weight_bytes(N, K, r)
    assert got == _weight_bytes_for_tile(N, K, r, tile)
    for other in (256, 192, 128):
        # another width that divides N would give a different blob whenever its scale atoms differ
        if other != tile and N % other == 0 and _weight_bytes_for_tile(N, K, r, other) != \
                _weight_bytes_for_tile(N, K, r, tile):
            assert got != _weight_bytes_for_tile(N, K, r, other)


def test_tile_width_override(L, monkeypatch):
    """SVDQ_N_TILE picks another valid width; an invalid one is ignored."""
    N, K, r = 768, 512, 32  # 768 = 3 x 256 = 4 x 192 = 6 x 128
    assert L.svdq_weight_bytes(N, K, r) == _weight_bytes_for_tile(N, K, r, 256)
    monkeypatch.setenv("SVDQ_N_TILE", "128")
    assert L.svdq_weight_bytes(N, K, r) == _weight_bytes_for_tile(N, K, r, 128)
    monkeypatch.setenv("SVDQ_N_TILE", "96")
    assert L.svdq_weight_bytes(N, K, r) == _weight_bytes_for_tile(N, K, r, 256)


def test_concat_lora_ranks():
    """A LoRA adapter extends the branch; the total rank must be one the kernels take."""
    import torch
    from bit_diffusion_transformer_svdquant_b200.prepare import concat_lora
    K, N = 64, 48
    prep = {"R": torch.zeros(N, K), "L1s": torch.zeros(K, 16, dtype=torch.bfloat16),
            "L2": torch.zeros(16, N, dtype=torch.bfloat16), "inv_lambda": torch.ones(K)}
    out = concat_lora(prep, torch.ones(K, 16), torch.full((16, N), 2.0))
    assert out["L1s"].shape == (K, 32) and out["L2"].shape == (32, N)
    assert out["L1s"].dtype == torch.bfloat16 and float(out["L1s"][0, 20]) == 1.0 and float(out["L2"][20, 0]) == 2.0
    assert torch.equal(out["L1s"][:, :16], prep["L1s"])
    with pytest.raises(ValueError):
        concat_lora(prep, torch.ones(K, 8), torch.ones(8, N))  # 16 + 8 = 24
    p0 = dict(prep, L1s=None, L2=None)
    assert concat_lora(p0, torch.ones(K, 16), torch.ones(16, N))["L1s"].shape == (K, 16)


# ---------------------------------------------------------------- row-wise FP8 variant (host logic)

def _up(x):
    return (x + 255) // 256 * 256


def test_fp8r_size_queries(L):
    N, K, r = 9216, 3072, 32
    want = _up(N * K) + _up(N * 4) + _up(K * 4) + _up(r * K * 2) + _up(2 * N * r * 2)
    assert L.svdq_fp8r_weight_bytes(N, K, r) == want
    assert L.svdq_fp8r_weight_bytes(N, 3000, r) == 0
    assert L.svdq_fp8r_weight_bytes(N, K, 24) == 0
    assert L.svdq_fp8r_weight_bytes(100, K, r) == 0
    M = 16896
    assert L.svdq_fp8r_act_bytes(M, K, r) == _up(M * K) + 2 * _up(M * 4) + _up(2 * M * r * 2)
    assert L.svdq_fp8r_act_bytes(0, K, r) == 0
    assert L.svdq_fp8r_act_bytes(M, K, 8) == 0


def test_fp8r_act_bind_layout(L):
    act = _lib.SvdqFp8rAct()
    base = 1 << 40
    M, K, r = 300, 512, 16
    nb = L.svdq_fp8r_act_bytes(M, K, r)
    assert L.svdq_fp8r_act_bind(M, K, r, ctypes.c_void_p(base), nb, ctypes.byref(act)) == 0
    assert act.M_pad == 384 and act.codes == base
    assert act.row_scale - act.codes == 384 * 512
    assert act.row_rscale - act.row_scale == _up(384 * 4) and act.U - act.row_rscale == _up(384 * 4)
    assert base + nb - act.U >= 2 * 384 * 16 * 2
    assert L.svdq_fp8r_act_bind(M, K, r, ctypes.c_void_p(base), nb - 1, ctypes.byref(act)) == 1
    assert L.svdq_fp8r_act_bind(M, K, r, ctypes.c_void_p(base + 16), nb, ctypes.byref(act)) == 2


def _fake_fp8r_pair(L):
    base = 1 << 40
    w = _lib.SvdqFp8rWeight(N=512, K=512, r=16, swiglu_interleaved=0, n_tile=256)
    for i, f in enumerate(("codes", "row_scale", "inv_lambda", "L1s_t", "L2_t")):
        setattr(w, f, base + (i << 20))
    act = _lib.SvdqFp8rAct()
    assert L.svdq_fp8r_act_bind(300, 512, 16, ctypes.c_void_p(base + (64 << 20)), 1 << 30, ctypes.byref(act)) == 0
    return w, act


@pytest.mark.parametrize("field,value", [("n_tile", 96), ("N", 640), ("r", 8), ("codes", None), ("row_scale", None),
                                         ("L2_t", None), ("M_pad", 512), ("M", -1), ("row_rscale", None), ("U", None)])
def test_fp8r_descriptor_checks_before_any_cuda_call(L, field, value):
    w, act = _fake_fp8r_pair(L)
    p = ctypes.c_void_p(1 << 41)
    tgt = act if field in ("M_pad", "M", "row_rscale", "U") else w
    setattr(tgt, field, value)
    assert L.svdq_fp8r_gemm(ctypes.byref(act), ctypes.byref(w), None, 0, p, 0, None) == 1, L.svdq_last_error()
    assert L.svdq_fp8r_quantize_act(p, ctypes.byref(w), ctypes.byref(act), None) == 1, L.svdq_last_error()
    if tgt is w:
        assert L.svdq_fp8r_export_weight(ctypes.byref(w), p, p, None) == 1
    else:
        assert L.svdq_fp8r_export_act(ctypes.byref(act), p, p, None) == 1
    assert b"descriptor" in L.svdq_last_error()


def test_fp8r_argument_checks_and_no_gpu(L):
    import torch
    w = _lib.SvdqFp8rWeight()
    p = ctypes.c_void_p(1 << 40)
    assert L.svdq_fp8r_pack_weight(None, p, p, p, 512, 512, 16, 0, p, 1 << 30, ctypes.byref(w), None) == 1
    assert L.svdq_fp8r_pack_weight(p, p, p, p, 500, 512, 16, 0, p, 1 << 30, ctypes.byref(w), None) == 2
    assert L.svdq_fp8r_pack_weight(p, p, p, p, 512, 512, 16, 0, p, 16, ctypes.byref(w), None) == 1  # dst too small
    fw, fa = _fake_fp8r_pair(L)
    fw.swiglu_interleaved = 1
    assert L.svdq_fp8r_gemm(ctypes.byref(fa), ctypes.byref(fw), None, 0, p, 0, None) == 1      # packed for SwiGLU
    fw.swiglu_interleaved = 0
    assert L.svdq_fp8r_gemm(ctypes.byref(fa), ctypes.byref(fw), None, 1, p, 0, None) == 1      # bias missing
    if torch.cuda.is_available():
        return
    st = L.svdq_fp8r_pack_weight(p, p, p, p, 512, 512, 16, 0, p, 1 << 30, ctypes.byref(w), None)
    assert st == 3, (st, L.svdq_last_error())
    assert L.svdq_fp8r_gemm(ctypes.byref(fa), ctypes.byref(fw), None, 0, p, 0, None) == 3


def test_prepare_layer_matches_oracle_preparation():
    """The torch offline helper against the oracle's preparation on the same data: identical
    smoothing reciprocals (bit for bit), the split identity W_hat = diag(lambda') L1s L2 + R to R's
    fp32 rounding, bf16 branch factors, and r = 0 giving exactly the oracle's R."""
    import numpy as np
    import torch
    from bit_diffusion_transformer_svdquant_b200.prepare import prepare_layer
    from oracle import svdquant
    rng = np.random.default_rng(3)
    M, K, N = 96, 256, 192
    X = rng.standard_normal((M, K))
    X[:, rng.choice(K, 4, replace=False)] *= 50
    X = svdquant.bf16_round(X)
    X[:, 7] = 0.0                                   # a silent channel: lambda = 1
    W = svdquant.bf16_round(rng.standard_normal((N, K)) / np.sqrt(K))
    Xt = torch.from_numpy(X.astype(np.float32)).to(torch.bfloat16)
    Wt = torch.from_numpy(W.astype(np.float32)).to(torch.bfloat16)
    ref = svdquant.prepare_layer(X, W, 16)
    got = prepare_layer(Xt, Wt, 16, torch.device("cpu"))
    assert np.array_equal(got["inv_lambda"].double().numpy(), ref["inv_lambda"])
    lam_p = 1.0 / got["inv_lambda"].double().numpy()
    W_hat = lam_p[:, None] * W.T                                           # [K, N]
    branch = (lam_p[:, None] * got["L1s"].double().numpy()) @ got["L2"].double().numpy()
    R = got["R"].double().numpy().T
    assert np.max(np.abs(W_hat - branch - R)) <= 2.0 ** -23 * np.max(np.abs(W_hat))
    assert got["L1s"].dtype == torch.bfloat16 and got["L2"].dtype == torch.bfloat16
    # the branch spans the same rank-16 space as the oracle's (signs of singular vectors may differ)
    ref_branch = (ref["lam_prime"][:, None] * ref["L1s"]) @ ref["L2"]
    assert np.max(np.abs(branch - ref_branch)) <= 2e-2 * np.max(np.abs(ref_branch))
    got0 = prepare_layer(Xt, Wt, 0, torch.device("cpu"))
    assert np.array_equal(got0["R"].double().numpy(), svdquant.prepare_layer(X, W, 0)["R"])


# ---------------------------------------------------------------- fused MLP chain (host logic)

def _fake_mlp(L):
    base = 1 << 40

    def weight(N, K, r, swiglu, n_tile, slot):
        w = _lib.SvdqWeight(N=N, K=K, r=r, swiglu_interleaved=swiglu, n_tile=n_tile)
        for i, f in enumerate(("codes", "scales", "g_w", "inv_lambda", "L1s_t", "L2_t")):
            setattr(w, f, base + (slot << 28) + (i << 20))
        return w

    def act(M, K, r, slot):
        a = _lib.SvdqAct()
        assert L.svdq_act_bind(M, K, r, ctypes.c_void_p(base + (slot << 28)), 1 << 27, ctypes.byref(a)) == 0
        return a

    return (act(300, 512, 16, 1), weight(1024, 512, 16, 1, 256, 2), weight(384, 512, 32, 0, 192, 3),
            act(300, 512, 32, 4))


def _call_mlp(L, a, w, wn, an, scratch_bytes=1 << 26):
    p = ctypes.c_void_p(1 << 41)
    return L.svdq_gemm_swiglu_quant(ctypes.byref(a), ctypes.byref(w), None, ctypes.byref(wn), p, ctypes.byref(an),
                                    p, scratch_bytes, None, None)


def test_mlp_scratch_bytes(L):
    assert L.svdq_mlp_scratch_bytes(4608, 32) == 8 * 4608 * 32 * 4
    assert L.svdq_mlp_scratch_bytes(300, 16) == 8 * 384 * 16 * 4
    assert L.svdq_mlp_scratch_bytes(300, 0) == 0 and L.svdq_mlp_scratch_bytes(0, 32) == 0


def test_mlp_fused_argument_checks(L):
    import torch
    a, w, wn, an = _fake_mlp(L)
    w.swiglu_interleaved = 0
    assert _call_mlp(L, a, w, wn, an) == 2                         # not a SwiGLU weight
    w.swiglu_interleaved, w.n_tile = 1, 128
    assert _call_mlp(L, a, w, wn, an) == 2                         # 256-wide tiles only
    w.n_tile = 256
    wn.K = 256
    an.K = 256
    assert _call_mlp(L, a, w, wn, an) == 1                         # next K != N / 2
    a, w, wn, an = _fake_mlp(L)
    wn.swiglu_interleaved = 1
    assert _call_mlp(L, a, w, wn, an) == 1                         # next layer packed for SwiGLU
    a, w, wn, an = _fake_mlp(L)
    assert _call_mlp(L, a, w, wn, an, scratch_bytes=1024) == 1     # scratch too small
    an2 = _lib.SvdqAct()
    assert L.svdq_act_bind(256, 512, 32, ctypes.c_void_p(1 << 44), 1 << 27, ctypes.byref(an2)) == 0
    assert _call_mlp(L, a, w, wn, an2) == 1                        # next act has another M
    a, w, wn, an = _fake_mlp(L)
    wn.r = 0
    an0 = _lib.SvdqAct()
    assert L.svdq_act_bind(300, 512, 0, ctypes.c_void_p(1 << 44), 1 << 27, ctypes.byref(an0)) == 0
    assert _call_mlp(L, a, w, wn, an0) == 2                        # next layer needs a branch rank
    if not torch.cuda.is_available():
        a, w, wn, an = _fake_mlp(L)
        assert _call_mlp(L, a, w, wn, an) == 3, L.svdq_last_error()  # well-formed: stops at the device


def test_binding_refuses_cpu_tensors():
    """No CPU fallback in the binding either: host tensors are refused before any library call."""
    import torch
    import bit_diffusion_transformer_svdquant_b200 as svdq
    R, inv = torch.zeros(128, 256), torch.ones(256)
    L1, L2 = torch.zeros(256, 16, dtype=torch.bfloat16), torch.zeros(16, 128, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="CUDA"):
        svdq.PackedWeight(R, L1, L2, inv)
    with pytest.raises(ValueError, match="CUDA"):
        svdq.Fp8rWeight(R, L1, L2, inv)
    with pytest.raises(ValueError, match="CUDA"):
        svdq.PackedWeight(R.double(), L1, L2, inv)          # and the wrong dtype


C_PROGRAM = r"""
#include <stddef.h>
#include <stdio.h>
#include "svdq.h"
int main(void) {
  svdq_act act;
  unsigned char* base = (unsigned char*)0 + ((size_t)1 << 40);
  size_t nb = svdq_act_bytes(300, 512, 16);
  svdq_status st = svdq_act_bind(300, 512, 16, base, nb, &act);
  svdq_weight w;
  float* p = (float*)((size_t)1 << 41);
  svdq_status st2 = svdq_pack_weight(p, (const uint16_t*)p, (const uint16_t*)p, p, 512, 512, 16, 0, p,
                                     (size_t)1 << 30, &w, NULL);
  printf("%d %zu %zu %zu %d %d %d %zu %zu %d %zu %zu %zu %zu %s\n", svdq_abi_version(),
         svdq_weight_bytes(9216, 3072, 32), nb, svdq_fp8r_weight_bytes(9216, 3072, 32), (int)st, act.M_pad,
         (int)(act.scales != NULL), svdq_mlp_scratch_bytes(4608, 32), sizeof(svdq_weight), (int)st2,
         sizeof(svdq_act), sizeof(svdq_fp8r_weight), sizeof(svdq_fp8r_act),
         offsetof(svdq_weight, tmap), svdq_status_str(st2));
  return 0;
}
"""


def test_header_is_plain_c_and_links(L, tmp_path):
    """include/svdq.h compiles as C99 and a C program links against libsvdq.so and runs its
    host-only calls; the answers agree with the ctypes binding, and a compute call without a GPU
    fails with SVDQ_ERR_CUDA."""
    import shutil
    import subprocess
    import torch
    gcc = shutil.which("gcc") or shutil.which("cc")
    if gcc is None:
        pytest.skip("no C compiler")
    src = tmp_path / "abi.c"
    src.write_text(C_PROGRAM)
    exe = tmp_path / "abi"
    libdir = os.path.dirname(_lib.LIB_PATH)
    r = subprocess.run([gcc, "-std=c99", "-Wall", "-Werror", "-pedantic", "-I", os.path.dirname(_lib.HEADER),
                        str(src), "-L", libdir, "-lsvdq", f"-Wl,-rpath,{libdir}", "-o", str(exe)],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert out.returncode == 0, out.stderr
    f = out.stdout.split()
    assert int(f[0]) == L.svdq_abi_version()
    assert int(f[1]) == L.svdq_weight_bytes(9216, 3072, 32)
    assert int(f[2]) == L.svdq_act_bytes(300, 512, 16)
    assert int(f[3]) == L.svdq_fp8r_weight_bytes(9216, 3072, 32)
    assert int(f[4]) == 0 and int(f[5]) == 384 and int(f[6]) == 1
    assert int(f[7]) == L.svdq_mlp_scratch_bytes(4608, 32)
    # the ctypes layouts match C's
    assert int(f[8]) == ctypes.sizeof(_lib.SvdqWeight)
    assert int(f[10]) == ctypes.sizeof(_lib.SvdqAct)
    assert int(f[11]) == ctypes.sizeof(_lib.SvdqFp8rWeight)
    assert int(f[12]) == ctypes.sizeof(_lib.SvdqFp8rAct)
    assert int(f[13]) == _lib.SvdqWeight.tmap.offset
    if not torch.cuda.is_available():
        assert int(f[9]) == 3                                    # SVDQ_ERR_CUDA: no fallback


def test_weight_bind_checks(L):
    """svdq_weight_bind (checkpoint reload): host checks first; a well-formed call stops at the
    device query without a GPU."""
    import torch
    w = _lib.SvdqWeight()
    p = ctypes.c_void_p(1 << 40)
    need = _weight_bytes_for_tile(768, 512, 32, 128)
    assert L.svdq_weight_bind(768, 512, 32, 0, 128, None, need, ctypes.byref(w)) == 1        # null blob
    assert L.svdq_weight_bind(768, 512, 32, 0, 96, p, need, ctypes.byref(w)) == 2            # bad n_tile
    assert L.svdq_weight_bind(640, 512, 32, 0, 256, p, need, ctypes.byref(w)) == 2           # 640 % 256
    assert L.svdq_weight_bind(768, 500, 32, 0, 128, p, need, ctypes.byref(w)) == 2           # K % 256
    assert L.svdq_weight_bind(768, 512, 32, 0, 128, ctypes.c_void_p((1 << 40) + 16), need, ctypes.byref(w)) == 2
    assert L.svdq_weight_bind(768, 512, 32, 0, 128, p, need - 1, ctypes.byref(w)) == 1       # blob too small
    if not torch.cuda.is_available():
        assert L.svdq_weight_bind(768, 512, 32, 0, 128, p, need, ctypes.byref(w)) == 3


@pytest.mark.parametrize("N,K,r,tile", [(768, 512, 32, 128), (768, 512, 32, 192), (768, 512, 32, 256),
                                        (9216, 3072, 32, 256), (384, 256, 0, 192), (640, 1024, 64, 128),
                                        (9216, 3072, 32, 384), (768, 256, 16, 384)])
def test_weight_bytes_tiled(L, N, K, r, tile):
    """The size query with an explicit tile width gives the layout of that width."""
    assert L.svdq_weight_bytes_tiled(N, K, r, tile) == _weight_bytes_for_tile(N, K, r, tile)


def test_weight_bytes_tiled_rejects(L):
    assert L.svdq_weight_bytes_tiled(768, 512, 32, 96) == 0       # not a tile width
    assert L.svdq_weight_bytes_tiled(640, 512, 32, 256) == 0      # 256 does not divide 640
    assert L.svdq_weight_bytes_tiled(768, 500, 32, 128) == 0      # K % 256
    assert L.svdq_weight_bytes_tiled(768, 512, 24, 128) == 0      # rank
    assert L.svdq_weight_bytes_tiled(1152, 512, 32, 384) == 0     # 384-wide needs 768 | N
    assert L.svdq_weight_bytes_tiled(384, 512, 32, 384) == 0


def test_wide_tile_only_without_swiglu(L):
    """The 384-wide tile: a blob of the 256-wide size, refused for a SwiGLU weight on re-bind."""
    import torch
    assert L.svdq_weight_bytes_tiled(9216, 3072, 32, 384) == L.svdq_weight_bytes_tiled(9216, 3072, 32, 256)
    w = _lib.SvdqWeight()
    p = ctypes.c_void_p(1 << 40)
    need = _weight_bytes_for_tile(768, 512, 32, 384)
    assert L.svdq_weight_bind(768, 512, 32, 1, 384, p, need, ctypes.byref(w)) == 2           # SwiGLU at 384
    assert L.svdq_weight_bind(1152, 512, 32, 0, 384, p, need, ctypes.byref(w)) == 2          # 768 does not divide N
    if not torch.cuda.is_available():
        assert L.svdq_weight_bind(768, 512, 32, 0, 384, p, need, ctypes.byref(w)) == 3


def test_from_state_checks_the_blob(L):
    """A checkpoint whose blob is not a contiguous 1-D uint8 tensor of exactly the packed size for its
    N, K, r and n_tile is refused before anything is copied to a device."""
    import torch
    N, K, r, t = 768, 512, 32, 128
    need = _weight_bytes_for_tile(N, K, r, t)
    base = {"abi": L.svdq_abi_version(), "N": N, "K": K, "r": r, "swiglu": False, "n_tile": t}
    bad = [
        torch.zeros(need, dtype=torch.int8),                       # dtype changed on save / load
        torch.zeros(need // 2, dtype=torch.int16),
        torch.zeros(2, need // 2, dtype=torch.uint8),              # not one-dimensional
        torch.zeros(2 * need, dtype=torch.uint8)[::2],             # not contiguous
        torch.zeros(need + 256, dtype=torch.uint8),                # another layer's size
        torch.zeros(need - 256, dtype=torch.uint8),
    ]
    for blob in bad:
        with pytest.raises(ValueError, match="checkpoint blob"):
            _lib.PackedWeight.from_state({**base, "blob": blob}, "cpu")
    # fields of another layer (n_tile 192 over the 128-wide blob: 4 x 2 scale atoms per K step
    # instead of 6 x 1) are refused too
    assert _weight_bytes_for_tile(N, K, r, 192) != need
    with pytest.raises(ValueError, match="checkpoint blob"):
        _lib.PackedWeight.from_state({**base, "n_tile": 192, "blob": torch.zeros(need, dtype=torch.uint8)}, "cpu")
