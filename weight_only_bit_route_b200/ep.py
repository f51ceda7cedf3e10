"""Expert-parallel MoE layer: one process per GPU, the routed experts split across the ranks.

The layer of "Step 5 Preview: 92 narrow layers, and a sparse indexer that scores blocks of 8" (The shape: 352
routed experts, top-8, one shared expert per token), split the way the DEP8 deployment of the same page (15
October) splits it: every rank keeps its own tokens (data parallel), the router and the shared expert are
replicated, and rank r owns the routed experts [r * E / N, (r + 1) * E / N).  Per call on each rank:

    1. route the rank's tokens (moe_route_topk);
    2. group the T * top_k slots by owning rank (moe_permute with the ranks as the buckets);
    3. all-to-all: each slot's token row, its expert (local to the owner) and its routing weight go to the owner,
       as one record per slot;
    4. the owner runs its experts on the rows it received, as a batch of single-slot tokens (moe_permute by local
       expert, moe_grouped_w4a16_swiglu, moe_grouped_w4a16_down with the weight by row, moe_unpermute_combine with
       top_k = 1, which puts the rows back in the order received);
    5. all-to-all back, into the order the slots were sent;
    6. the shared expert on the rank's own tokens, and moe_unpermute_combine with the inverse of step 2's grouping
       (slot -> position in the returned rows): y[t] = shared[t] + sum_j of token t's returned rows.

Every step of the layer runs in the library's kernels; this module marshals arguments and moves rows between
ranks with torch.distributed (NCCL over NVLink on GPUs, gloo on CPU).  The send records are gathered, and the
(expert, weight) pairs appended, with torch indexing: data movement for the exchange, no arithmetic of the
layer.  The collective is the stock all-to-all: rows cross the fabric once each way, and no multicast of any
kind is used.  Each row's result is independent of which other rows share its tile, so on one rank the layer
reproduces moe_layer_decode bit for bit.

The split sizes of an all-to-all are host values, so each call reads the per-rank slot counts back to the host
once (after step 2) and the returned counts once (after the counts' exchange).  A rank whose batch is above
max_tokens still takes part in the counts' exchange (with counts of -1), and then every rank raises ValueError, so
an oversized batch on one rank ends the call on all of them instead of leaving the others in a collective.
"""
import torch
import torch.distributed as dist

from . import moe


class CudaOps:
    """The layer's steps on this rank's GPU, through the C ABI."""

    def __init__(self, gate, up, down, router_w, router_bias, top_k, shared, max_tokens, world):
        self.gate, self.up, self.down = gate, up, down
        self.router_w, self.router_bias, self.k, self.shared = router_w, router_bias, top_k, shared
        E, H = router_w.shape
        F, e_local = gate.out_dim, gate.E
        # route + owner grouping of up to max_tokens tokens; the experts of up to world * max_tokens * k rows.
        # (moe_workspace_bytes sizes a whole layer, which needs top_k <= E: the owner grouping, with the ranks
        # as its buckets, and the shared expert, E = 1, take a layer of top_k experts, which covers them.)
        dev = router_w.device
        self.ws_route = moe.workspace(max_tokens, H, E, F, top_k, device=dev)
        self.ws_owner = moe.workspace(max_tokens, 128, max(world, top_k), 128, top_k, device=dev)
        rows = max(world, 1) * max_tokens * top_k
        self.ws_experts = moe.workspace(rows, H, e_local, F, 1, device=dev)
        self.ws_shared = moe.workspace(max_tokens, H, top_k, F, top_k, device=dev) if shared else None

    def route(self, x):
        return moe.route_topk(x, self.router_w, self.router_bias, self.k, self.ws_route)

    def group(self, owner, world):
        return moe.permute(owner, world, self.ws_owner)

    def experts(self, xr, er, wr):
        R = xr.shape[0]
        if R == 0:
            return torch.empty_like(xr)
        off, rs, sr = moe.permute(er.view(R, 1), self.gate.E, self.ws_experts)
        h = moe.grouped_swiglu(xr, off, rs, 1, self.gate, self.up, R, self.ws_experts)
        yp = moe.grouped_down(h, off, rs, wr, self.down, self.ws_experts)
        return moe.unpermute_combine(yp, sr, R, 1)

    def shared_expert(self, x):
        if not self.shared:
            return None
        T = x.shape[0]
        so = torch.tensor([0, T], dtype=torch.int32, device=x.device)
        srs = torch.arange(T, dtype=torch.int32, device=x.device) * self.k
        hs = moe.grouped_swiglu(x, so, srs, self.k, self.shared[0], self.shared[1], T, self.ws_shared)
        return moe.grouped_down(hs, so, srs, None, self.shared[2], self.ws_shared)

    def combine(self, y_back, slot_pos, T, shared_out):
        return moe.unpermute_combine(y_back, slot_pos, T, self.k, shared_out)


class ExpertParallelMoE:
    """The routed experts [rank * E / world, (rank + 1) * E / world) of a layer on this rank.

    gate, up, down: this rank's experts only (moe.Bank with E / world experts); router_w (fp32 [E, H]),
    router_bias and shared (a (gate, up, down) tuple of E = 1 BF16 banks, or None) are the whole layer's,
    replicated.  max_tokens bounds the tokens of one call on any rank.  ops replaces the step implementations
    (tests run the collectives on CPU ranks with reference steps); by default the steps are the library's
    kernels on this rank's GPU."""

    def __init__(self, gate, up, down, router_w, top_k=8, router_bias=None, shared=None, group=None,
                 max_tokens=64, ops=None):
        self.group = group
        self.world = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        E = router_w.shape[0]
        if E % self.world or gate.E * self.world != E:
            raise ValueError(f"{E} experts do not split into {self.world} ranks of {gate.E}")
        self.E, self.e_per_rank, self.k, self.max_tokens = E, gate.E, top_k, max_tokens
        self.ops = ops if ops is not None else CudaOps(gate, up, down, router_w, router_bias, top_k, shared,
                                                       max_tokens, self.world)

    def _a2a(self, out, inp, out_split, in_split):
        dist.all_to_all_single(out, inp, out_split, in_split, group=self.group)

    def forward(self, x):
        """x: bf16 [T, H] (this rank's tokens, T <= max_tokens) -> y: bf16 [T, H]."""
        T, H = x.shape
        k, world = self.k, self.world
        dev = x.device
        # A batch above max_tokens is refused on every rank: the refusing rank sends counts of -1 in the counts'
        # exchange (which every rank takes), and every rank raises after it, so none is left waiting for a peer.
        refused = T > self.max_tokens
        if refused:
            send_counts = torch.full((world,), -1, dtype=torch.int64, device=dev)
        else:
            ids, w = self.ops.route(x)                                 # [T, k] expert ids, weights
            owner = torch.div(ids, self.e_per_rank, rounding_mode="floor").to(torch.int32)
            off, order, slot_pos = self.ops.group(owner, world)      # slots by owner; slot -> send position
            send_counts = (off[1:] - off[:-1]).to(torch.int64)
        recv_counts = torch.empty_like(send_counts)
        self._a2a(recv_counts, send_counts, None, None)
        sc, rc = send_counts.tolist(), recv_counts.tolist()
        if refused:
            raise ValueError(f"T = {T} exceeds max_tokens = {self.max_tokens}")
        if min(rc) < 0:
            raise ValueError(f"rank(s) {[r for r in range(world) if rc[r] < 0]} refused a batch above max_tokens")
        R = int(sum(rc))
        order_l = order.to(torch.int64)
        # one exchange for rows and their metadata: each record is the token row's bytes followed by the
        # slot's local expert and routing weight bits (an int32 pair)
        nb = H * x.element_size()
        meta = torch.stack([ids.view(-1).index_select(0, order_l) - owner.view(-1).index_select(0, order_l)
                            * self.e_per_rank,
                            w.view(-1).index_select(0, order_l).view(torch.int32)], dim=1)
        send = torch.empty(order_l.numel(), nb + 8, dtype=torch.uint8, device=dev)
        send[:, :nb] = x.index_select(0, torch.div(order_l, k, rounding_mode="floor")).view(torch.uint8)
        send[:, nb:] = meta.contiguous().view(torch.uint8)
        recv = torch.empty(R, nb + 8, dtype=torch.uint8, device=dev)
        self._a2a(recv, send, rc, sc)
        recv_x = recv[:, :nb].contiguous().view(x.dtype)
        recv_meta = recv[:, nb:].contiguous().view(torch.int32)
        er = recv_meta[:, 0].contiguous()
        wr = recv_meta[:, 1].contiguous().view(torch.float32)
        y_recv = self.ops.experts(recv_x, er, wr)                    # [R, H], received order
        y_back = torch.empty(T * k, H, dtype=x.dtype, device=dev)
        self._a2a(y_back.view(torch.uint8), y_recv.contiguous().view(torch.uint8), sc, rc)
        return self.ops.combine(y_back, slot_pos, T, self.ops.shared_expert(x))
