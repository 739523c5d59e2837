"""The C-ABI library builds, loads without a GPU, exports every entry point include/svdq.h declares,
and its host-side logic (size queries, layouts, argument checks) behaves; no compute call is made."""
import ctypes

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


def test_no_gpu_fails_loudly(L):
    """Valid arguments on a machine without a usable GPU: a CUDA error status, not a fallback."""
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    w = _lib.SvdqWeight()
    p = ctypes.c_void_p(1 << 40)
    st = L.svdq_pack_weight(p, p, p, p, 512, 512, 16, 0, p, 1 << 30, ctypes.byref(w), None)
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
