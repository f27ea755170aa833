"""Block-sharded data parallelism (segment 16, Lemma 2) on CPU: the owner
plan from the C library, and the reduce-scatter / owner step / all-gather
plumbing of ShardedShampoo over gloo with world sizes 2 and 3.

The ranks' local optimizer here is the fp64 oracle on CPU tensors (the CUDA
library needs a GPU); what is under test is the plumbing around it: after
every step each rank must hold exactly the weights that one oracle over all
parameters produces from the mean of the ranks' gradients.
"""
import itertools
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

from shampoo_second_order_b200 import _lib as L
from shampoo_second_order_b200 import workloads as wl


def free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


# --------------------------------------------------------------------------
# the plan
# --------------------------------------------------------------------------
def solo_cost(shape, b, interval):
    _, cost = L.shampoo_plan_shards([shape], b, interval, 1)
    return cost[0]


def test_plan_covers_every_parameter_deterministically():
    c = wl.CONFIGS["resnet50_b128"]
    a, ca = L.shampoo_plan_shards(c["shapes"], c["block_size"], c["root_interval"], 8)
    b, cb = L.shampoo_plan_shards(c["shapes"], c["block_size"], c["root_interval"], 8)
    assert a == b and ca == cb
    assert sorted(set(a)) == list(range(8))
    costs = [solo_cost(s, c["block_size"], c["root_interval"]) for s in c["shapes"]]
    for r in range(8):   # the per-rank cost is the sum of its parameters' costs
        assert abs(sum(x for x, o in zip(costs, a) if o == r) - ca[r]) <= 1e-9 * ca[r]


@pytest.mark.parametrize("seed,ranks", [(0, 2), (1, 3), (2, 2), (3, 3)])
def test_plan_is_within_the_lpt_bound_of_the_best_split(seed, ranks):
    """Longest-processing-time first is within (4/3 - 1/(3m)) of the optimal
    makespan (Graham 1969); checked against brute force on 7 parameters."""
    rng = np.random.default_rng(seed)
    shapes = [(int(rng.integers(1, 300)), int(rng.integers(1, 300))) for _ in range(7)]
    owner, load = L.shampoo_plan_shards(shapes, 64, 10, ranks)
    costs = [solo_cost(s, 64, 10) for s in shapes]
    best = min(max(sum(c for c, o in zip(costs, assign) if o == r) for r in range(ranks))
               for assign in itertools.product(range(ranks), repeat=len(shapes)))
    assert max(load) <= (4 / 3 - 1 / (3 * ranks)) * best * (1 + 1e-12)


def test_plan_rejects_bad_arguments():
    with pytest.raises(L.ShampooError):
        L.shampoo_plan_shards([(4, 4)], 64, 10, 0)
    with pytest.raises(L.ShampooError):
        L.shampoo_plan_shards([(0, 4)], 64, 10, 2)


# --------------------------------------------------------------------------
# the sharded step over gloo
# --------------------------------------------------------------------------
class OracleLocal:
    """The per-rank optimizer, as the fp64 oracle over CPU tensors."""

    def __init__(self, shapes, b, beta2, eps, graft, mu):
        from oracle import ShampooOracle
        self.o = ShampooOracle(shapes, b, beta2, eps, 4, graft, mu)

    def update_stats(self, grads):
        self.o.update_stats([g.double().numpy() for g in grads])

    def compute_roots(self):
        self.o.compute_roots()

    def apply(self, params, grads, lr):
        new = self.o.apply([p.double().numpy() for p in params], [g.double().numpy() for g in grads], lr)
        for p, w in zip(params, new):
            p.copy_(__import__("torch").from_numpy(w).to(p.dtype))


SHAPES = [(70, 40), (33,), (40, 90), (8, 8), (130,), (64, 64), (1, 50)]
CFG = dict(b=32, beta2=0.95, eps=1e-2, graft=1, mu=0.5, lr=0.05, steps=5, interval=2)


def _rank_grads(rank, t, dtype="f32"):
    return wl.make_grads(SHAPES, 100 + rank, t, 1e-1, dtype)


def _worker(rank, world, port, q, dtype="f32"):
    import torch
    import torch.distributed as dist
    from datetime import timedelta
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    from oracle import ShampooOracle
    from shampoo_second_order_b200.sharded import ShardedShampoo
    c = CFG
    opt = ShardedShampoo(SHAPES, c["b"], c["beta2"], c["eps"], graft=c["graft"], momentum=c["mu"],
                         grad_dtype=dtype, root_interval=c["interval"],
                         make_local=lambda sh: OracleLocal(sh, c["b"], c["beta2"], c["eps"], c["graft"], c["mu"]))
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    ref = ShampooOracle(SHAPES, c["b"], c["beta2"], c["eps"], 4, c["graft"], c["mu"])
    W0 = wl.make_params(SHAPES, 5)
    W = [torch.from_numpy(w.astype(np.float32)) for w in W0]
    Wr = [w.astype(np.float32).astype(np.float64) for w in W0]
    worst = 0.0
    for t in range(c["steps"]):
        mine = _rank_grads(rank, t, dtype)
        # the exact mean of the ranks' gradients (bf16 values held exactly)
        mean = [sum(_rank_grads(r, t, dtype)[i].astype(np.float64) for r in range(world)) / world
                for i in range(len(SHAPES))]
        roots = t % c["interval"] == 0
        opt.step(W, [torch.from_numpy(g).to(tdt) for g in mine], c["lr"], roots)
        Wr = ref.step(Wr, mean, c["lr"], roots)
        for w, r_ in zip(W, Wr):
            d = np.abs(w.double().numpy() - r_).max() / max(np.abs(r_).max(), 1e-30)
            worst = max(worst, d)
    # every rank holds the same weights
    flat = torch.cat([w.reshape(-1) for w in W])
    other = [torch.empty_like(flat) for _ in range(world)]
    dist.all_gather(other, flat)
    same = all(torch.equal(other[0], x) for x in other)
    dist.barrier()
    dist.destroy_process_group()
    q.put((rank, worst, same, opt.mine, opt.collective_bytes_per_step()))


@pytest.mark.parametrize("world,dtype", [(2, "f32"), (3, "f32"), (2, "bf16"), (3, "bf16")])
def test_sharded_step_matches_one_oracle_on_mean_gradients(world, dtype):
    """bf16 gradients are summed in float32: a bf16 reduction would round
    each partial sum to 8 bits and miss the 1e-6 bar by orders of magnitude."""
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q, dtype)) for r in range(world)]
    for p in procs:
        p.start()
    out = [q.get(timeout=300) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    owned = []
    for rank, worst, same, mine, nbytes in out:
        assert worst <= 1e-6, (rank, worst)     # float32 weights and float32 gradient sums
        assert same
        assert nbytes > 0
        owned += mine
    assert sorted(owned) == list(range(len(SHAPES)))   # every parameter has exactly one owner


def _dying_worker(rank, world, port, q):
    import torch
    import torch.distributed as dist
    from datetime import timedelta
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=10))
    from shampoo_second_order_b200.sharded import ShardedShampoo
    c = CFG
    opt = ShardedShampoo(SHAPES, c["b"], c["beta2"], c["eps"], graft=c["graft"], momentum=c["mu"],
                         root_interval=c["interval"],
                         make_local=lambda sh: OracleLocal(sh, c["b"], c["beta2"], c["eps"], c["graft"], c["mu"]))
    W = [torch.from_numpy(w.astype(np.float32)) for w in wl.make_params(SHAPES, 5)]
    g = [torch.from_numpy(x) for x in _rank_grads(rank, 0)]
    opt.step(W, g, c["lr"], True)                 # one good step together
    if rank == 1:
        q.put((rank, "died"))
        q.close()
        q.join_thread()                            # the message is out before the process goes
        os._exit(3)                                # leaves between steps, nothing in flight
    import time
    t0 = time.time()
    try:
        opt.step(W, g, c["lr"], False)
        q.put((rank, "no error"))
    except Exception as e:                         # the collective reports the missing rank
        q.put((rank, "error after %.1f s: %s" % (time.time() - t0, type(e).__name__)))
    q.close()
    q.join_thread()
    os._exit(0)


def test_sharded_step_reports_a_dead_rank():
    """A rank that leaves between steps: the survivor's next reduce-scatter
    ends with an error from the process group (within its 10 s timeout), not
    a hang."""
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = free_port()
    procs = [ctx.Process(target=_dying_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = dict(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
    assert out[1] == "died"
    assert out[0].startswith("error after"), out[0]
    assert float(out[0].split()[2]) < 60
