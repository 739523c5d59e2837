"""A discrete-event model of the barrier protocol of the row-wise FP8 GEMM (gemm_kernel in
csrc/svdq_fp8r.cuh), checked on the host, in the manner of test_fused_protocol_model.py: the
producer, the MMA issuer, the relay warp and the eight epilogue warps of both CTAs of a pair replay
their barrier traffic in the kernel's order; copies landing and MMA commits completing arrive late
and in random order. The protocol differs from the NVFP4 GEMM's in its two accumulator buffers
(used alternately, so one tile's epilogue overlaps the next tile's MMAs) and in the relay warp
that reports each ring slot's arrival in its CTA to the issuer's barrier (two arrivals per slot).
Checked: no deadlock, no stray arrival, waits on exactly the completion they mean, and no resource
(ring stage, a slot's data in both CTAs, an accumulator buffer) used before its previous user is
done. Removing any one wait must make the model fail."""
import random

import pytest

SYNC_BUFS = 4
WAITS = ["producer.empty", "issuer.acce", "issuer.sync", "relay.full", "relay.release", "epi.accf"]


class Barrier:
    def __init__(self, name, count):
        self.name, self.count, self.pending, self.completed = name, count, count, 0

    def arrive(self, n=1):
        self.pending -= n
        assert self.pending >= 0, f"{self.name}: more arrivals than its count in one phase"
        if self.pending == 0:
            self.completed += 1
            self.pending = self.count


def run_model(n_tiles, r, k_iters, stages, seed, skip=()):
    rng = random.Random(seed)
    slots = (r + 31) // 32 + k_iters
    B = {}

    def bar(name, count):
        B[name] = Barrier(name, count)

    for c in (0, 1):
        for s in range(stages):
            bar(f"full{c}.{s}", 1)
            bar(f"empty{c}.{s}", 1)
        for a in range(2):
            bar(f"accf{c}.{a}", 1)
    for a in range(2):
        bar(f"acce{a}", 16)             # 8 epilogue warps x 2 CTAs
    for b in range(SYNC_BUFS):
        bar(f"sync{b}", 2)              # the relay warp of each CTA
    done = lambda name: B[name].completed  # noqa: E731
    in_flight = []

    def wait(tag, name, index):
        if tag in skip:
            return
        while (B[name].completed & 1) == (index & 1):
            yield name
        assert B[name].completed == index + 1, \
            f"{name}: wait for completion #{index} passed at completed = {B[name].completed}"

    def producer(c):
        uses = [0] * stages
        stage = 0
        for _ in range(n_tiles * slots):
            yield from wait("producer.empty", f"empty{c}.{stage}", uses[stage] - 1)
            assert done(f"empty{c}.{stage}") >= uses[stage], "ring stage refilled while its MMAs read it"
            uses[stage] += 1
            in_flight.append(f"full{c}.{stage}")
            stage = (stage + 1) % stages

    def issuer():
        stage, sb, g = 0, 0, 0
        sync_uses = [0] * SYNC_BUFS
        for t in range(n_tiles):
            a, use = t & 1, t >> 1
            yield from wait("issuer.acce", f"acce{a}", use - 1)
            assert done(f"acce{a}") >= use, "accumulator buffer overwritten before its epilogue read it"
            for _ in range(slots):
                yield from wait("issuer.sync", f"sync{sb}", sync_uses[sb])
                sync_uses[sb] += 1
                for c in (0, 1):
                    assert done(f"full{c}.{stage}") >= g // stages + 1, "MMA before a CTA's copy landed"
                for c in (0, 1):
                    in_flight.append(f"empty{c}.{stage}")
                stage = (stage + 1) % stages
                sb = (sb + 1) % SYNC_BUFS
                g += 1
            for c in (0, 1):
                in_flight.append(f"accf{c}.{a}")

    def relay(c):
        full_uses = [0] * stages
        released = [0] * stages
        stage, sb, n = 0, 0, 0
        for _ in range(n_tiles * slots):
            yield from wait("relay.full", f"full{c}.{stage}", full_uses[stage])
            full_uses[stage] += 1
            if n >= SYNC_BUFS:
                ps = (stage - SYNC_BUFS) % stages
                yield from wait("relay.release", f"empty{c}.{ps}", released[ps])
                released[ps] += 1
            B[f"sync{sb}"].arrive()
            n += 1
            stage = (stage + 1) % stages
            sb = (sb + 1) % SYNC_BUFS

    def epilogue(c):
        for t in range(n_tiles):
            a, use = t & 1, t >> 1
            yield from wait("epi.accf", f"accf{c}.{a}", use)
            assert done(f"accf{c}.{a}") >= use + 1, "accumulator read before its MMAs completed"
            B[f"acce{a}"].arrive()

    live = {"issuer": issuer()}
    for c in (0, 1):
        live[f"producer{c}"] = producer(c)
        live[f"relay{c}"] = relay(c)
        for w in range(8):
            live[f"epi{c}.{w}"] = epilogue(c)

    for _ in range(1_000_000):
        if not live:
            break
        waiting = {}
        for k in rng.sample(sorted(live), len(live)):
            try:
                waiting[k] = next(live[k])
            except StopIteration:
                del live[k]
        if live and not in_flight and all(waiting.get(k) is not None for k in live):
            still = {}
            for k in list(live):
                try:
                    still[k] = next(live[k])
                except StopIteration:
                    del live[k]
            if live and not in_flight and all(v is not None for v in still.values()):
                raise AssertionError(f"deadlock: {still}")
        rng.shuffle(in_flight)
        for _ in range(rng.randint(0, len(in_flight))):
            B[in_flight.pop()].arrive()
    assert not live, "model did not finish"
    while in_flight:
        B[in_flight.pop()].arrive()
    for name, b in B.items():
        assert b.pending == b.count, f"{name}: {b.count - b.pending} stray arrivals at the end"
    return True


# the kernel's ring depths: 6 stages for 256- and 192-wide tiles, 8 for 128-wide ones
@pytest.mark.parametrize("stages", [6, 8])
@pytest.mark.parametrize("n_tiles", [1, 2, 3, 7])
@pytest.mark.parametrize("r,k_iters", [(32, 2), (64, 1), (0, 4), (16, 24)])
def test_fp8r_protocol_model(stages, n_tiles, r, k_iters):
    for seed in range(5):
        assert run_model(n_tiles, r, k_iters, stages, seed)


@pytest.mark.parametrize("skipped", WAITS)
def test_every_wait_is_needed(skipped):
    for n_tiles in (3, 7):
        for r, k_iters in ((32, 2), (0, 4), (16, 24)):
            for seed in range(20):
                try:
                    run_model(n_tiles, r, k_iters, 6, seed, skip={skipped})
                except AssertionError:
                    return
    pytest.fail(f"removing the wait {skipped} went unnoticed")
