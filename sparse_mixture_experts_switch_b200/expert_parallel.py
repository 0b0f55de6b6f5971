"""Expert-parallel Switch-FFN layer over a torch.distributed group.

Plumbing only: buffers, peer pointers and the two collectives between the
library's three expert-parallel calls (include/switch_moe.h, "Expert
parallelism").  Every step of the layer itself -- routing, global slot
ranks, the row exchange, the expert GEMMs, the combine on the token's home
rank and the loss -- runs in the CUDA library.

The split follows "Switch Transformers: scaling to trillion-parameter
models", section "Distributed Implementation and the Three Parallelisms"
(expert-parallelism row): each rank owns N / G experts and its own T
tokens; tokens travel to their expert's rank and the results travel back.
The G ranks' batches form one routing group in rank order, so capacity,
drops and the loss are those of one GPU holding all G * T tokens.

One forward step on every rank:

    switch_ep_route      -> this rank's exchange record
    all-gather of the records (rank order)
    switch_ep_dispatch   -> rows stored into the owners' receive buffers
    barrier              (every rank's rows have landed)
    switch_ep_experts    -> outputs stored on the tokens' home ranks
    barrier              (every rank's outputs are complete)

The receive buffers and the outputs are written by other ranks' kernels,
so they live in memory every rank's GPU can reach: by default PyTorch's
symmetric memory over NVLink (`peer_alloc` replaces it, e.g. for tests).
"""
import torch
import torch.distributed as dist

from . import switch_moe as _sm


def symmetric_peer_alloc(group):
    """Allocator of peer-reachable buffers through PyTorch's symmetric memory:
    returns (this rank's tensor, the G ranks' device addresses)."""
    import torch.distributed._symmetric_memory as symm_mem

    def alloc(shape, dtype, device):
        t = symm_mem.empty(shape, dtype=dtype, device=device)
        try:
            h = symm_mem.rendezvous(t, group)
        except (TypeError, RuntimeError):
            h = symm_mem.rendezvous(t, group.group_name)
        return t, list(h.buffer_ptrs)
    return alloc


class ExpertParallelSwitch:
    """The layer forward, expert parallel over `group` (default: WORLD).

    T: tokens per rank (equal on every rank); n_experts: N for the whole
    layer (N % G == 0); this rank's experts are rank * N / G ..
    (rank + 1) * N / G - 1.  `lib` is the binding (switch_moe by default).
    """

    def __init__(self, T, d_model, d_ff, n_experts, capacity_factor, alpha=0.01, flags=0,
                 group=None, device=None, peer_alloc=None, lib=None):
        self.lib = lib or _sm
        self.group = group if group is not None else dist.group.WORLD
        self.G = dist.get_world_size(self.group)
        self.rank = dist.get_rank(self.group)
        self.device = torch.device(device) if device is not None else torch.device(
            "cuda", torch.cuda.current_device())
        self.T, self.d_model, self.n_experts = T, d_model, n_experts
        self.cfg = self.lib.config(T, d_model, d_ff, n_experts, capacity_factor, alpha=alpha,
                                   flags=flags)
        self.ep = self.lib.ep(self.G, self.rank)
        ws_b, rec_b, recv_b = self.lib.switch_ep_sizes(self.cfg, self.ep)
        self.record_bytes = rec_b
        u8 = dict(dtype=torch.uint8, device=self.device)
        self.ws = torch.zeros(max(ws_b, 1), **u8)
        self.record = torch.zeros(max(rec_b, 16), **u8)
        self.records = torch.zeros(self.G * max(rec_b, 16), **u8)
        alloc = peer_alloc or symmetric_peer_alloc(self.group)
        self.recv, self.recv_peers = alloc((max(recv_b, 256),), torch.uint8, self.device)
        self.out, self.out_peers = alloc((max(T, 1), d_model), torch.bfloat16, self.device)
        self.counts = torch.zeros(n_experts, dtype=torch.int32, device=self.device)
        self.loss = torch.zeros(1, dtype=torch.float32, device=self.device)
        self._flag = torch.zeros(1, dtype=torch.int32, device=self.device)

    @property
    def experts(self):
        """Range of the experts this rank owns."""
        e = self.n_experts // self.G
        return range(self.rank * e, (self.rank + 1) * e)

    def _all_gather_records(self):
        try:
            dist.all_gather_into_tensor(self.records, self.record, group=self.group)
        except (RuntimeError, NotImplementedError, AttributeError):
            dist.all_gather(list(self.records.view(self.G, -1).unbind(0)), self.record,
                            group=self.group)

    def _barrier(self):
        # stream-ordered: completes once every rank's earlier kernels have
        dist.all_reduce(self._flag, group=self.group)

    def forward(self, x, w_r, b_r, w1_local, w2_local, idx=None, gate=None):
        """x [T, d_model] bf16 on this rank; w_r / b_r the whole router;
        w1_local / w2_local this rank's experts' weights.  Returns this rank's
        output [T, d_model] (a view of the peer-reachable output buffer), the
        loss (device scalar) and the counts of the whole batch."""
        lib = self.lib
        lib.switch_ep_route(self.cfg, self.ep, x, w_r, b_r, idx, gate, self.record, self.ws)
        self._all_gather_records()
        lib.switch_ep_dispatch(self.cfg, self.ep, x, self.records, self.recv_peers, self.out,
                               self.counts, self.loss, self.ws)
        self._barrier()
        lib.switch_ep_experts(self.cfg, self.ep, w1_local, w2_local, self.recv, self.out_peers,
                              self.ws)
        self._barrier()
        return self.out[:self.T], self.loss, self.counts
