"""Expert-parallel MXFP4 MoE layer over a torch.distributed process group.

agentlenshq "Transformers ... GPT-OSS" (ja), section "Expert parallel (EP)":
the MoE experts are distributed over the GPUs, which lowers the per-GPU load;
"Tricks from OpenAI gpt-oss you can use with transformers" (summary),
section 8: the shards compute in parallel and a collective gathers the
results.  Here the E experts are split in G contiguous ranges, rank r holding
experts [r E/G, (r + 1) E/G) in MXFP4.  Every rank brings its own tokens and
router logits (data parallel over tokens); one forward is

  1. route (moe_route) and group the T k routed rows by expert (moe_permute).
     Experts of one rank are contiguous, so the rows are grouped by
     destination rank as well: rank r's share is the count sum of its experts;
  2. exchange the per-expert counts (all_to_all), then the rows themselves
     (all_to_all of x_perm: each destination receives, from every source, its
     experts' rows in expert order);
  3. on the receiving rank, regroup the rows from all sources by local expert
     (moe_permute with k = 1, stable, so source order is kept inside an
     expert), run the grouped expert MLP (moe_expert_mlp) and put the results
     back in arrival order (moe_combine with k = 1 and weight 1, which copies
     each bf16 row exactly);
  4. send the results back (all_to_all with the reversed splits): they land in
     the sender's x_perm order, which is the y_perm order of the one-GPU layer;
  5. combine on the token's owner (moe_combine), the same weighted sum, in the
     same order, as the one-GPU layer.

Every arithmetic step runs in the library's CUDA kernels (``LibraryOps``).
The host computes only the split sizes from the per-expert counts, which it
copies from the device (the sent and the received counts: the two
synchronisations of a forward).  The rows travel as int32 pairs of bf16 bit
patterns, which any backend moves unchanged.  A different ``ops`` object
supplies the four compute calls for tests that run the exchange on CPU ranks;
the default is the CUDA library and there is no other default.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np
import torch
import torch.distributed as dist


@dataclass
class LocalExperts:
    """The MXFP4 weights of the experts one rank holds: ``first`` is the
    global index of its first expert, ``count`` how many it holds.  Codes and
    scales as ``moe_expert_mlp`` takes them: wgu [count][2F][D/2] +
    [count][2F][D/32], wdn [count][D][F/2] + [count][D][F/32]."""
    first: int
    count: int
    wgu_q: torch.Tensor
    wgu_s: torch.Tensor
    wdn_q: torch.Tensor
    wdn_s: torch.Tensor


def expert_range(E: int, world: int, rank: int) -> tuple[int, int]:
    """Contiguous expert range [first, first + count) of ``rank``: the E
    experts split as evenly as possible, lower ranks taking the remainder."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("bad rank / world")
    if E < world:
        raise ValueError(f"{E} experts cannot be split over {world} ranks")
    base, extra = divmod(E, world)
    first = rank * base + min(rank, extra)
    return first, base + (1 if rank < extra else 0)


def send_splits(counts: np.ndarray, E: int, world: int) -> list[int]:
    """Rows this rank sends to each rank: the sum of its per-expert counts
    over each rank's expert range."""
    out = []
    for r in range(world):
        f, c = expert_range(E, world, r)
        out.append(int(counts[f:f + c].sum()))
    return out


def received_layout(counts_from: np.ndarray) -> np.ndarray:
    """Local expert index of every received row, in arrival order, from the
    [world][local experts] matrix of counts the sources sent: source 0's rows
    first, each source's rows in local-expert order."""
    world, n_local = counts_from.shape
    ids = [np.repeat(np.arange(n_local, dtype=np.int32), counts_from[s]) for s in range(world)]
    return np.concatenate(ids) if ids else np.zeros(0, dtype=np.int32)


class LibraryOps:
    """The compute calls of an expert-parallel forward, on the CUDA library."""

    def __init__(self, device, stream=None):
        import mxfp4_quantised_mixture_b200 as moe

        self.moe = moe
        self.device = torch.device(device)
        self.stream = stream

    def route(self, logits: torch.Tensor, k: int):
        T = logits.shape[0]
        idx = torch.empty((T, k), dtype=torch.int32, device=self.device)
        w = torch.empty((T, k), dtype=torch.float32, device=self.device)
        self.moe.moe_route(logits, k, idx, w, self.stream)
        return idx, w

    def permute(self, idx: torch.Tensor, x: torch.Tensor, E: int, d_ff: int):
        T, k = idx.shape
        D = x.shape[1]
        sh = self.moe.make_shape(T, E, k, D, d_ff)
        counts = torch.empty(E, dtype=torch.int32, device=self.device)
        offsets = torch.empty(E + 1, dtype=torch.int32, device=self.device)
        sorted_slot = torch.empty(T * k, dtype=torch.int32, device=self.device)
        slot_pos = torch.empty(T * k, dtype=torch.int32, device=self.device)
        x_perm = torch.empty((T * k, D), dtype=torch.bfloat16, device=self.device)
        self.moe.moe_permute(idx, x, sh, counts, offsets, sorted_slot, slot_pos, x_perm, None,
                             self.stream)
        return counts, offsets, slot_pos, x_perm

    def expert_mlp(self, x_perm: torch.Tensor, offsets: torch.Tensor, ex: LocalExperts,
                   d_ff: int):
        R, D = x_perm.shape
        sh = self.moe.make_shape(R, ex.count, 1, D, d_ff)
        h = torch.empty((R, d_ff), dtype=torch.bfloat16, device=self.device)
        y = torch.empty((R, D), dtype=torch.bfloat16, device=self.device)
        ws = self.moe.alloc_workspace(sh, self.moe.WS_EXPERT_MLP, self.device)
        self.moe.moe_expert_mlp(x_perm, offsets, sh, ex.wgu_q, ex.wgu_s, ex.wdn_q, ex.wdn_s, h, y,
                                ws, self.stream)
        return y

    def combine(self, y_perm: torch.Tensor, slot_pos: torch.Tensor, w: torch.Tensor, E: int,
                d_ff: int):
        T, k = w.shape
        D = y_perm.shape[1]
        out = torch.empty((T, D), dtype=torch.bfloat16, device=self.device)
        self.moe.moe_combine(y_perm, slot_pos, w, self.moe.make_shape(T, E, k, D, d_ff), out,
                             self.stream)
        return out

    def to_host(self, t: torch.Tensor) -> np.ndarray:
        return t.cpu().numpy()

    def from_host(self, a: np.ndarray) -> torch.Tensor:
        return torch.from_numpy(a).to(self.device)


def _exchange(t: torch.Tensor, send: list[int], recv: list[int], group) -> torch.Tensor:
    """all_to_all of bf16 rows [n][D]: ``send[r]`` leading rows go to rank r,
    ``recv[r]`` rows arrive from rank r.  The rows travel as int32 pairs of
    bit patterns (D is even), which every backend moves unchanged."""
    D = t.shape[1]
    if t.shape[0] == 0:  # nothing to send (an empty tensor may carry any strides)
        bits = torch.empty((0, D // 2), dtype=torch.int32, device=t.device)
    else:
        bits = t.contiguous().view(torch.int32)
    out = torch.empty((sum(recv), D // 2), dtype=torch.int32, device=t.device)
    dist.all_to_all_single(out, bits, output_split_sizes=recv, input_split_sizes=send, group=group)
    return out.view(torch.bfloat16)


def ep_layer_forward(x: torch.Tensor, logits: torch.Tensor, k: int, E: int, d_ff: int,
                     local: LocalExperts, ops=None, group=None) -> torch.Tensor:
    """One expert-parallel MoE layer: x [T][D] bf16 and logits [T][E] fp32 of
    this rank's tokens -> out [T][D] bf16, the same rows the one-GPU layer
    gives for these tokens over all E experts.  Every rank of ``group`` calls
    it (collective), each with its own T (0 allowed)."""
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    first, count = expert_range(E, world, rank)
    if (first, count) != (local.first, local.count):
        raise ValueError(f"rank {rank} holds experts [{local.first}, +{local.count}), "
                         f"the split needs [{first}, +{count})")
    if ops is None:
        ops = LibraryOps(x.device)
    D = x.shape[1]

    # 1. route and group the routed rows by expert (hence by destination)
    idx, w = ops.route(logits, k)
    counts, _, slot_pos, x_perm = ops.permute(idx, x, E, d_ff)
    counts_h = ops.to_host(counts).astype(np.int64)
    send = send_splits(counts_h, E, world)

    # 2. per-expert counts to the experts' owners (each owner's range is a
    #    contiguous run of the counts), then the rows
    n_local = [expert_range(E, world, r)[1] for r in range(world)]
    cnt_recv = torch.empty(world * count, dtype=torch.int32, device=counts.device)
    dist.all_to_all_single(cnt_recv, counts, output_split_sizes=[count] * world,
                           input_split_sizes=n_local, group=group)
    counts_from = ops.to_host(cnt_recv).astype(np.int64).reshape(world, count)
    recv = [int(c) for c in counts_from.sum(axis=1)]
    x_recv = _exchange(x_perm, send, recv, group)

    # 3. regroup by local expert, grouped MLP, back to arrival order
    R = sum(recv)
    if R > 0:
        ids = ops.from_host(received_layout(counts_from).reshape(R, 1))
        _, offsets_l, slot_pos_l, x_local = ops.permute(ids, x_recv, count, d_ff)
        y_local = ops.expert_mlp(x_local, offsets_l, local, d_ff)
        ones = ops.from_host(np.ones((R, 1), dtype=np.float32))
        y_recv = ops.combine(y_local, slot_pos_l, ones, count, d_ff)
    else:
        y_recv = x_recv.new_empty((0, D))

    # 4. results back to the senders, in their x_perm order
    y_perm = _exchange(y_recv, recv, send, group)

    # 5. weighted combine on the token's owner
    return ops.combine(y_perm, slot_pos, w, E, d_ff)
