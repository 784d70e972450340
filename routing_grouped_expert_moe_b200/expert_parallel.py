"""Expert-parallel forward of the MoE layer: one process per GPU, rank r of G
owning experts [r*E/G, (r+1)*E/G).

"ops-transformer 算子精讲：昇腾 NPU 上的注意力机制与融合算子实现" ch.5: with the
experts spread over devices, routing costs two all-to-all exchanges, one that
sends each token's hidden state to the devices of its chosen experts and one
that brings the expert outputs back.  "ops-transformer 仓库 - MoE 算子优化实战",
core principles, point 2 (sparse-computation optimisation): expert
parallelism, with one aggregated all-to-all instead of point-to-point messages.

Every rank runs the layer on its own tokens (its own capacity and drops, as
one single-device call would) and the results equal, row for row, what one
single-device forward of those tokens over all E experts gives:

  1. route and permute the local tokens over all E experts (the permuted rows
     come out grouped by expert, hence by owning rank);
  2. exchange the per-expert kept-row counts (all-to-all, E/G int32 per pair);
  3. exchange the rows (all-to-all with per-rank splits); the received block
     is ordered [source rank][local expert];
  4. regroup it by local expert (a k = 1 permute, stable, so sources stay in
     rank order inside an expert), run the grouped FFN, and put the outputs
     back in received order (a k = 1 unpermute);
  5. the reverse all-to-all returns each output row to the rank and the row
     slot its input came from, and the local combine sums the gated rows.

Rows travel as raw bytes, so any storage type crosses unchanged.  The split
sizes are read on the host, since all-to-all with uneven splits takes them
there: the count exchange runs on the device first, so one device-to-host
read per forward brings back this rank's offsets and the counts it receives.

The per-rank compute steps are the C ABI's kernels (`CudaSteps`); torch.distributed
(NCCL between GPUs) carries the two exchanges.

With overlap=True (and at least two experts per rank) the local experts form
two groups, A = the first half and B = the rest, and the rows move as
point-to-point messages per group, following the same pages' point that
expert parallelism lets communication overlap computation: B's rows travel
while A's experts run, and A's outputs travel back while B's experts run.
Every (rank, local expert) block is a message of its own, a slice of the
sender's expert-ordered rows, and lands at its place in an expert-major
buffer (local expert, then source rank), so the group's rows go to the
grouped FFN without a regroup and its outputs go back block by block; a
rank's blocks for itself are copied locally.
"""
from __future__ import annotations

import numpy as np
import torch
import torch.distributed as dist


def split_rows(offsets: np.ndarray, world: int) -> np.ndarray:
    """Rows of the expert-ordered block destined to each rank: rank d owns experts
    [d*E/G, (d+1)*E/G), whose rows run from offsets[d*E/G] to offsets[(d+1)*E/G]."""
    offsets = np.asarray(offsets, dtype=np.int64)
    E = offsets.size - 1
    if E % world:
        raise ValueError(f"{E} experts do not split evenly over {world} ranks")
    el = E // world
    return np.array([offsets[(d + 1) * el] - offsets[d * el] for d in range(world)],
                    dtype=np.int64)


def local_expert_ids(recv_kept: np.ndarray) -> np.ndarray:
    """Local expert id of every received row.  recv_kept[s, j] rows of local expert j
    arrive from source rank s, sources in rank order, experts in order inside each."""
    recv_kept = np.asarray(recv_kept, dtype=np.int64)
    G, el = recv_kept.shape
    return np.repeat(np.tile(np.arange(el, dtype=np.int32), G), recv_kept.reshape(-1))


class CudaSteps:
    """The per-rank compute steps, each one call into the C ABI on the current stream."""

    def __init__(self):
        from routing_grouped_expert_moe_b200 import binding
        self.B = binding

    def route(self, x, w_gate, gate_bias, top_k):
        return self.B.route(x, w_gate, gate_bias, top_k)

    def permute(self, x, idx, E, capacity_factor):
        p = self.B.permute(idx, E, capacity_factor, x=x)
        return p["x_perm"], p["offsets"], p["row_map"]

    def grouped_ffn(self, x_rows, offsets, w1, w3, w2, act):
        return self.B.grouped_ffn(offsets, w1, w3, w2, act, x_perm=x_rows)

    def unpermute(self, y, row_map):
        return self.B.unpermute_combine(y, None, row_map)

    def combine(self, y, gate, row_map):
        return self.B.unpermute_combine(y, gate, row_map)

    def to_host(self, t):
        return t.cpu().numpy()

    def from_host(self, a, like):
        return torch.from_numpy(np.ascontiguousarray(a)).to(like.device)


def _bytes(t: torch.Tensor) -> torch.Tensor:
    """The rows of a contiguous [n, H] tensor as [n, H * element size] bytes."""
    return t.view(torch.uint8)


def _post(msgs, me, group, tag):
    """Start one point-to-point round.  msgs: (peer, send, recv) triples in an order
    both sides of every pair derive alike from the exchanged counts (send: a
    contiguous byte view going to the peer, recv: one the peer fills; None when
    empty, so both sides skip the same messages).  Messages between two ranks
    are matched in the order they are posted; a rank's blocks for itself are
    copied locally.  Returns the pending requests."""
    ops = []
    for peer, snd, rcv in msgs:
        if peer == me:
            if rcv is not None:
                rcv.copy_(snd)
            continue
        gpeer = peer if group is None else dist.get_global_rank(group, peer)
        if snd is not None:
            ops.append(dist.P2POp(dist.isend, snd, gpeer, group, tag))
        if rcv is not None:
            ops.append(dist.P2POp(dist.irecv, rcv, gpeer, group, tag))
    return dist.batch_isend_irecv(ops) if ops else []


def _wait(works):
    for w in works:
        w.wait()


def _rows(buf, a, b):
    return _bytes(buf[a:b]) if b > a else None


def _overlapped_experts(steps, x_perm, offsets, recv_kept, w1, w3, w2, act, G, el, me,
                        group, y_back):
    """Rows out, experts, rows back, in two expert groups that overlap (see the module
    docstring); fills y_back (rows in the order of x_perm).  Each (rank, local
    expert) block travels as a message of its own and lands in expert order
    (local expert, then source rank), so the received rows go to the grouped FFN
    as they are and its outputs go back block by block: no regroup."""
    H = x_perm.shape[1]
    halves = [(0, el // 2), (el // 2, el)]
    layouts = []                       # per group: block starts [group size, G], segment starts
    bufs = []                          # per group: the received rows, expert-major
    pending = []
    keep = []                          # outputs still being sent back
    for gi, (j0, j1) in enumerate(halves):
        rk = recv_kept[:, j0:j1]                       # [source, local expert of the group]
        sizes = rk.T.reshape(-1)                       # expert-major: (j, s)
        starts = np.concatenate([[0], np.cumsum(sizes)]).astype(np.int64)
        pos = starts[:-1].reshape(j1 - j0, G)
        seg = np.concatenate([[0], np.cumsum(rk.sum(axis=0))]).astype(np.int64)
        buf = x_perm.new_empty(int(starts[-1]), H)
        msgs = []
        for p in range(G):             # per peer: its experts of the group, in order
            for j in range(j0, j1):
                a = int(pos[j - j0, p])
                msgs.append((p, _rows(x_perm, int(offsets[p * el + j]),
                                      int(offsets[p * el + j + 1])),
                             _rows(buf, a, a + int(rk[p, j - j0]))))
        pending.append(_post(msgs, me, group, tag=gi))
        layouts.append((rk, pos, seg))
        bufs.append(buf)
    for gi, (j0, j1) in enumerate(halves):
        _wait(pending[gi])             # this group's rows are here; the next may still travel
        rk, pos, seg = layouts[gi]
        buf = bufs[gi]
        if buf.shape[0] > 0:
            sl = slice(j0, j1)
            off = steps.from_host(seg.astype(np.int32), buf)
            y_grp = steps.grouped_ffn(buf, off, None if w1 is None else w1[sl],
                                      None if w3 is None else w3[sl],
                                      None if w2 is None else w2[sl], act)
        else:
            y_grp = buf
        msgs = []
        for p in range(G):
            for j in range(j0, j1):
                a = int(pos[j - j0, p])
                msgs.append((p, _rows(y_grp, a, a + int(rk[p, j - j0])),
                             _rows(y_back, int(offsets[p * el + j]),
                                   int(offsets[p * el + j + 1]))))
        pending.append(_post(msgs, me, group, tag=2 + gi))
        keep.append(y_grp)
    for w in pending[len(halves):]:
        _wait(w)
    del keep


def ep_forward(x, w_gate, gate_bias, w1_local, w3_local, w2_local, top_k: int,
               capacity_factor: float, act: str, num_experts: int, group=None, steps=None,
               overlap: bool = False):
    """The layer's output [T, H] for this rank's tokens x [T, H].

    w_gate [H, E] (and gate_bias [E]) are the whole router, the same on every
    rank; w1_local / w3_local [E/G, H, F] and w2_local [E/G, F, H] are this rank's
    experts (w3_local None for GELU).  Every rank of `group` must call this
    together with the same E, top_k, act, storage type and overlap (T may
    differ).  overlap=True splits the exchanges in two expert groups so that
    transfers overlap the expert GEMMs (needs E/G >= 2; otherwise ignored)."""
    steps = steps or CudaSteps()
    G = dist.get_world_size(group)
    E = int(num_experts)
    if E % G:
        raise ValueError(f"{E} experts do not split evenly over {G} ranks")
    el = E // G
    if w1_local is not None and w1_local.shape[0] != el:
        raise ValueError(f"w1_local holds {w1_local.shape[0]} experts, expected {el}")
    T, H = x.shape
    dev = x.device

    # 1. route and permute this rank's tokens over all E experts
    if T > 0:
        idx, gate = steps.route(x, w_gate, gate_bias, top_k)
        x_perm, offsets_d, row_map = steps.permute(x, idx, E, capacity_factor)
    else:
        gate = row_map = None
        x_perm = x.new_empty(0, H)
        offsets_d = torch.zeros(E + 1, dtype=torch.int32, device=dev)

    # 2. kept-row counts per (destination, expert), exchanged on the device; then
    # the forward's one host read brings back this rank's offsets and the counts
    # it receives together (an uneven all-to-all takes its split sizes on the host)
    offsets_d = offsets_d.to(torch.int32)
    kept_d = offsets_d[1:] - offsets_d[:-1]
    recv_kept_d = torch.empty(E, dtype=torch.int32, device=dev)
    dist.all_to_all_single(recv_kept_d, kept_d, group=group)
    both = steps.to_host(torch.cat([offsets_d, recv_kept_d])).astype(np.int64)
    offsets, recv_kept = both[:E + 1], both[E + 1:].reshape(G, el)
    send = split_rows(offsets, G)
    R = int(offsets[E])
    recv = recv_kept.sum(axis=1)
    R_in = int(recv.sum())

    if overlap and el >= 2:
        # 3-5 in two expert groups whose transfers overlap the other group's experts
        y_back = x.new_empty(max(R, 1), H)
        _overlapped_experts(steps, x_perm, offsets, recv_kept, w1_local, w3_local, w2_local,
                            act, G, el, dist.get_rank(group), group, y_back)
        if T == 0:
            return x.new_empty(0, H)
        return steps.combine(y_back, gate, row_map)

    # 3. the rows, to the ranks that own their experts
    x_in = x.new_empty(R_in, H)
    dist.all_to_all_single(_bytes(x_in), _bytes(x_perm[:R]), output_split_sizes=recv.tolist(),
                           input_split_sizes=send.tolist(), group=group)

    # 4. regroup by local expert, run the experts, restore the received order
    if R_in > 0:
        ids = steps.from_host(local_expert_ids(recv_kept).reshape(R_in, 1), x_in)
        x_loc, off_loc, map_loc = steps.permute(x_in, ids, el, 0.0)
        y_loc = steps.grouped_ffn(x_loc, off_loc, w1_local, w3_local, w2_local, act)
        y_in = steps.unpermute(y_loc, map_loc)
    else:
        y_in = x.new_empty(0, H)

    # 5. outputs back to the rows they came from, then the gated sum per token
    y_back = x.new_empty(max(R, 1), H)
    dist.all_to_all_single(_bytes(y_back[:R]), _bytes(y_in), output_split_sizes=send.tolist(),
                           input_split_sizes=recv.tolist(), group=group)
    if T == 0:
        return x.new_empty(0, H)
    return steps.combine(y_back, gate, row_map)
