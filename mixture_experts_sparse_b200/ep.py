"""Expert parallelism: the experts of one MoE layer spread over G GPUs.

"From Switch Transformer to GLaM", section All-to-All: each device holds some
of the experts; a dispatch all-to-all sends every token to the device of its
expert and a combine all-to-all brings the expert output back.  Here every GPU
keeps its own batch as its own routing group (its capacity, its aux loss), so
its output is exactly the one-GPU layer forward of that batch, while the
expert FFN of expert e runs on GPU e // E (E = N / G) with only that GPU's
weights.  All the arithmetic runs in libmoe_b200's kernels; this module holds
buffers, the pointer tables that let a kernel store into another GPU's
buffers, and the order of the calls:

    route + slot claim (moe_route, moe_dispatch)  ->  all-gather kept [N]
    ->  moe_ep_layout  ->  moe_ep_dispatch (peer stores)  ->  barrier
    ->  moe_ep_expert_ffn (results stored back from the GEMM epilogue)
    ->  barrier  ->  top-2: moe_combine

`comm` supplies the two exchanges: LocalComm runs the G GPUs' phases one
after another in one process on one device (every "peer" buffer is then on
that device and the barriers are plain stream order); DistComm is one process
per GPU over torch.distributed, with the peers' buffers mapped through CUDA
IPC and the barriers as one-element all-reduces on the stream.
"""
import torch

from . import native as nat

WEIGHT_KEYS = ("w1", "b1", "w3", "b3", "w2", "b2")


def a2a_bytes(kept_all, rank, d_model, elem_bytes):
    """Bytes GPU `rank` sends over the links in one forward: its kept rows for
    other GPUs' experts (dispatch) plus the result rows it returns to other
    GPUs (combine).  kept_all: [G][N] kept rows per GPU and expert."""
    G = len(kept_all)
    N = len(kept_all[0])
    E = N // G
    sent = sum(int(kept_all[rank][e]) for e in range(N) if e // E != rank)
    returned = sum(int(kept_all[s][e]) for s in range(G) if s != rank for e in range(rank * E, (rank + 1) * E))
    return (sent + returned) * d_model * elem_bytes


def layout_host(kept_all, rank):
    """Host restatement of moe_ep_layout (tests): (dst_start [N], recv_offsets [E + 1])."""
    G = len(kept_all)
    N = len(kept_all[0])
    E = N // G
    tot = [sum(int(kept_all[s][e]) for s in range(G)) for e in range(N)]
    start = [sum(tot[(e // E) * E:e]) for e in range(N)]
    dst = [start[e] + sum(int(kept_all[s][e]) for s in range(rank)) for e in range(N)]
    recv = [start[rank * E + j] for j in range(E)] + [start[rank * E + E - 1] + tot[rank * E + E - 1]]
    return dst, recv


class LocalComm:
    """The G GPUs' phases one after another in one process (one device)."""

    def all_gather(self, tensors):
        return torch.stack(list(tensors))

    def barrier(self):
        pass


class DistComm:
    """One process per GPU over torch.distributed (this process: one rank)."""

    def __init__(self, group=None):
        import torch.distributed as dist
        self.dist = dist
        self.group = group
        self.flag = None

    def all_gather(self, tensors):
        (t,) = tensors
        dev = t.device
        if self.dist.get_backend(self.group) != "nccl":   # gloo gathers host tensors
            t = t.cpu()
        parts = [torch.empty_like(t) for _ in range(self.dist.get_world_size(self.group))]
        self.dist.all_gather(parts, t.contiguous(), group=self.group)
        return torch.stack(parts).to(dev)

    def barrier(self):
        if self.dist.get_backend(self.group) == "nccl":
            if self.flag is None:
                self.flag = torch.zeros(1, dtype=torch.int32, device="cuda")
            self.dist.all_reduce(self.flag, group=self.group)   # stream-ordered: later kernels wait for every rank
        else:
            torch.cuda.synchronize()
            self.dist.barrier(group=self.group)


class EpRank:
    """One GPU of an expert-parallel layer: its batch of T tokens (its own
    routing group of capacity C), its E = N / G experts and its receive buffers."""

    def __init__(self, G, rank, T, d_model, d_ff, n_experts, top_k, C, dtype, act, w_r, b_r, local_weights,
                 alpha=1e-2, device="cuda"):
        if n_experts % G:
            raise ValueError("the experts must split evenly over the GPUs")
        self.G, self.rank, self.T, self.N, self.k = G, rank, T, n_experts, top_k
        self.E = n_experts // G
        self.cfg = nat.config(T, d_model, d_ff, n_experts, top_k, C, dtype, act, alpha)
        self.ws = nat.new_workspace(self.cfg, device)
        self.w_r, self.b_r = w_r, b_r
        self.w = local_weights                 # this GPU's experts: w1 [E, d_ff, d] ...
        act_t = torch.bfloat16 if dtype == "bf16" else torch.float32
        i32, f32, f64 = torch.int32, torch.float32, torch.float64
        N, k, d = n_experts, top_k, d_model
        R = max(1, min(k * T, N * C))
        dev = dict(device=device)
        self.idx = torch.empty(T, k, dtype=i32, **dev)
        self.gate = torch.empty(T, k, dtype=f32, **dev)
        self.pos = torch.empty(T, k, dtype=i32, **dev)
        self.drop = torch.empty(T, k, dtype=torch.uint8, **dev)
        self.counts = torch.empty(k, N, dtype=i32, **dev)
        self.kept = torch.empty(N, dtype=i32, **dev)
        self.offsets = torch.empty(N + 1, dtype=i32, **dev)
        self.row_token = torch.empty(R, dtype=i32, **dev)
        self.row_gate = torch.empty(R, dtype=f32, **dev)
        self.f = torch.empty(N, dtype=f64, **dev)
        self.P = torch.empty(N, dtype=f64, **dev)
        self.aux = torch.empty(1, dtype=f64, **dev)
        self.out = torch.empty(T, d, dtype=act_t, **dev)
        self.ye = torch.zeros(R, d, dtype=act_t, **dev) if top_k == 2 else None
        Rr = max(1, nat.moe_ep_recv_rows(self.cfg, G))
        self.recv_x = torch.empty(Rr, d, dtype=act_t, **dev)
        self.recv_rank = torch.empty(Rr, dtype=i32, **dev)
        self.recv_row = torch.empty(Rr, dtype=i32, **dev)
        self.recv_gate = torch.empty(Rr, dtype=f32, **dev)
        self.dst_start = torch.empty(N, dtype=i32, **dev)
        self.recv_offsets = torch.empty(self.E + 1, dtype=i32, **dev)
        nb = nat.moe_ep_workspace_bytes(self.cfg, G)
        if nb == 0:
            raise ValueError("invalid expert-parallel configuration")
        self.ws_ep = torch.empty(nb, dtype=torch.uint8, **dev)
        nat.check(nat.moe_workspace_init(self.ws_ep))
        self.tables = None
        self._peer_refs = []                   # keeps IPC mappings alive

    # buffers other GPUs store into, in table order
    def shared(self):
        return dict(recv_x=self.recv_x, recv_rank=self.recv_rank, recv_row=self.recv_row,
                    recv_gate=self.recv_gate, dest=self.out if self.k == 1 else self.ye)

    def set_tables(self, per_rank):
        """per_rank: for every GPU s (in order), the dict of its shared buffers
        as this process sees them (its own, or IPC-mapped)."""
        def table(key):
            return torch.tensor([p[key].data_ptr() for p in per_rank], dtype=torch.int64, device=self.out.device)
        self.tables = {key: table(key) for key in ("recv_x", "recv_rank", "recv_row", "recv_gate", "dest")}

    def route_and_claim(self, x):
        nat.check(nat.moe_route(self.cfg, x, self.w_r, self.b_r, self.idx, self.gate, None, self.f, self.P,
                                self.aux, self.ws))
        nat.check(nat.moe_dispatch(self.cfg, x, self.idx, self.gate, self.pos, self.drop, self.counts, self.kept,
                                   self.offsets, self.row_token, self.row_gate, None, self.ws))
        return self.kept

    def layout(self, kept_all):
        nat.check(nat.moe_ep_layout(self.G, self.rank, self.N, kept_all, self.dst_start, self.recv_offsets))

    def send(self, x):
        t = self.tables
        nat.check(nat.moe_ep_dispatch(self.cfg, self.G, self.rank, x, self.offsets, self.row_token, self.row_gate,
                                      self.drop, self.dst_start, t["recv_x"], t["recv_rank"], t["recv_row"],
                                      t["recv_gate"], self.out))

    def experts(self):
        w = self.w
        nat.check(nat.moe_ep_expert_ffn(self.cfg, self.G, self.recv_x, self.recv_offsets, w["w1"], w.get("b1"),
                                        w.get("w3"), w.get("b3"), w["w2"], w.get("b2"), self.recv_rank,
                                        self.recv_row, self.recv_gate, self.tables["dest"], self.ws_ep))

    def combine(self):
        if self.k == 2:
            nat.check(nat.moe_combine(self.cfg, self.ye, self.idx, self.pos, self.drop, self.gate, self.offsets,
                                      self.out))
        return self.out


def link_local(ranks):
    """Pointer tables for GPUs emulated in one process on one device."""
    shared = [r.shared() for r in ranks]
    for r in ranks:
        r.set_tables(shared)


def link_ipc(rank_obj, group=None):
    """Pointer tables across processes: every rank exports its shared buffers
    through CUDA IPC (torch's tensor reduction), all-gathers the handles and
    maps the peers' buffers."""
    import torch.distributed as dist
    from torch.multiprocessing.reductions import reduce_tensor
    mine = {key: reduce_tensor(t) for key, t in rank_obj.shared().items()}
    world = dist.get_world_size(group)
    got = [None] * world
    dist.all_gather_object(got, mine, group=group)
    per_rank = []
    for s, handles in enumerate(got):
        if s == rank_obj.rank:
            per_rank.append(rank_obj.shared())
            continue
        peer = {key: fn(*args) for key, (fn, args) in handles.items()}
        rank_obj._peer_refs.append(peer)
        per_rank.append(peer)
    rank_obj.set_tables(per_rank)


def ep_forward(ranks, xs, comm):
    """One expert-parallel forward of the given GPUs (ranks[i] on input xs[i]).
    Returns their outputs (each the one-GPU forward of its own batch)."""
    kept = [r.route_and_claim(x) for r, x in zip(ranks, xs)]
    kept_all = comm.all_gather(kept)
    for r in ranks:
        r.layout(kept_all)
    for r, x in zip(ranks, xs):
        r.send(x)
    comm.barrier()                      # every GPU's rows are in their experts' receive buffers
    for r in ranks:
        r.experts()
    comm.barrier()                      # every result row is back on its source GPU
    return [r.combine() for r in ranks]
