"""The expert-parallel layer's exchange on CPU ranks (gloo): experts split
over 2 to 4 ranks, each rank with its own tokens (one with none), and every
rank's output rows equal to the oracle's one-process layer over all tokens,
bit for bit (agentlenshq "Transformers ... GPT-OSS" (ja), section "Expert
parallel (EP)").

The compute calls (route, permute, expert MLP, combine) are the oracle's,
injected as the ``ops`` object, so what runs here is the exchange itself: the
split sizes, the two all_to_all rounds in each direction, the regrouping on
the expert's owner and the order the results come back in.
"""
import os
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from mxfp4_quantised_mixture_b200 import ep  # noqa: E402


class OracleOps:
    """The four compute calls of ep_layer_forward on the CPU oracle (tests
    only); bf16 tensors are CPU torch.bfloat16, weights CPU uint8."""

    def __init__(self):
        import oracle

        self.o = oracle

    @staticmethod
    def _u16(t):
        return t.contiguous().view(torch.int16).numpy().view(np.uint16)

    @staticmethod
    def _bf16(a):
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16)

    def route(self, logits, k):
        idx, w = self.o.route(logits.numpy(), k)
        return torch.from_numpy(idx), torch.from_numpy(w)

    def permute(self, idx, x, E, d_ff):
        k = idx.shape[1]
        counts, offsets, sorted_slot, slot_pos = self.o.permute(idx.numpy(), E)
        x_perm = self.o.gather(self._u16(x), sorted_slot, k)
        return (torch.from_numpy(counts), torch.from_numpy(offsets), torch.from_numpy(slot_pos),
                self._bf16(x_perm))

    def expert_mlp(self, x_perm, offsets, ex, d_ff):
        _, y = self.o.expert_mlp(self._u16(x_perm), offsets.numpy(), ex.wgu_q.numpy(),
                                 ex.wgu_s.numpy(), ex.wdn_q.numpy(), ex.wdn_s.numpy(),
                                 want_h=False)
        return self._bf16(y)

    def combine(self, y_perm, slot_pos, w, E, d_ff):
        k = w.shape[1]
        return self._bf16(self.o.combine(self._u16(y_perm), slot_pos.numpy(), w.numpy(), k))

    def to_host(self, t):
        return t.numpy()

    def from_host(self, a):
        return torch.from_numpy(np.ascontiguousarray(a))


def _problem(T, D, F, E, seed, skew):
    import oracle
    import synthetic as syn

    x = syn.normal_bf16(seed, 1, (T, D), sigma=1.0)
    lg = np.random.default_rng(seed).standard_normal((T, E)).astype(np.float32)
    if skew:  # most tokens prefer the first experts: uneven loads, idle owners
        lg += np.linspace(6.0, 0.0, E, dtype=np.float32)
    gu = syn.normal_bf16(seed, 3, (E, 2 * F, D), sigma=0.02)
    dn = syn.normal_bf16(seed, 4, (E, D, F), sigma=0.02)
    gq, gs = oracle.quantize_experts(gu)
    dq, ds = oracle.quantize_experts(dn)
    return x, lg, gq, gs, dq, ds


def _worker(rank, world, port, case, q):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime

    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        import oracle

        T, D, F, E, k, seed, skew, bounds = case
        x, lg, gq, gs, dq, ds = _problem(T, D, F, E, seed, skew)
        a, b = bounds[rank], bounds[rank + 1]
        first, count = ep.expert_range(E, world, rank)
        local = ep.LocalExperts(first, count,
                                *(torch.from_numpy(np.ascontiguousarray(t[first:first + count]))
                                  for t in (gq, gs, dq, ds)))
        x_r = torch.from_numpy(x[a:b].view(np.int16)).view(torch.bfloat16)
        out = ep.ep_layer_forward(x_r, torch.from_numpy(lg[a:b]), k, E, F, local, ops=OracleOps())
        got = out.view(torch.int16).numpy().view(np.uint16)
        want = oracle.layer_forward(x, lg, k, gq, gs, dq, ds)[a:b]
        q.put((rank, bool(np.array_equal(got, want)), int(got.shape[0])))
    except Exception:  # reported to the parent, which fails the test
        import traceback

        q.put((rank, traceback.format_exc(), -1))
    finally:
        dist.destroy_process_group()


def _run(world, case):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29600 + (os.getpid() * 7 + world * 131) % 2000
    procs = [ctx.Process(target=_worker, args=(r, world, port, case, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=300) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    return sorted(res)


@pytest.mark.parametrize("world,case", [
    # world, (T, D, F, E, k, seed, skew, token bounds per rank)
    (2, (37, 128, 128, 8, 4, 1, False, [0, 20, 37])),
    (3, (41, 128, 192, 8, 4, 2, False, [0, 10, 10, 41])),   # rank 1 has no tokens; 8 = 3 + 3 + 2
    (2, (33, 128, 128, 16, 8, 3, True, [0, 1, 33])),        # skewed: a rank's experts may idle
    (4, (24, 256, 128, 4, 1, 4, False, [0, 6, 12, 18, 24])),  # one expert per rank, k = 1
])
def test_ep_layer_equals_one_process_layer(world, case):
    for rank, ok, n in _run(world, case):
        assert ok is True, (rank, ok)
        bounds = case[-1]
        assert n == bounds[rank + 1] - bounds[rank]


def test_expert_ranges_tile_the_experts():
    for E in (1, 4, 8, 32, 33, 128):
        for world in range(1, min(E, 9) + 1):
            spans = [ep.expert_range(E, world, r) for r in range(world)]
            assert spans[0][0] == 0
            for (f0, c0), (f1, _) in zip(spans, spans[1:]):
                assert f1 == f0 + c0
            assert sum(c for _, c in spans) == E
            assert max(c for _, c in spans) - min(c for _, c in spans) <= 1
    with pytest.raises(ValueError):
        ep.expert_range(2, 3, 0)


def test_send_splits_and_received_layout():
    counts = np.array([3, 0, 2, 5, 1, 4, 0, 2])
    assert ep.send_splits(counts, 8, 3) == [5, 10, 2]   # experts 0-2, 3-5, 6-7
    got = ep.received_layout(np.array([[2, 0, 1], [0, 3, 1]]))
    assert got.tolist() == [0, 0, 2, 1, 1, 1, 2]
    assert ep.received_layout(np.zeros((2, 3), dtype=np.int64)).size == 0
