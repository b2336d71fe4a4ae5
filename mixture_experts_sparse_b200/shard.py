"""One routing group split into contiguous shards (one per GPU).

Capacity is per routing group and claims follow token order over the group,
so a shard needs, per (rank, expert), the number of claims made before its own
tokens.  The only exchange is an all-gather of every shard's claim counts
([k, N] int32, a few hundred bytes) and, for the aux loss, of every shard's
f, P and token count.  Everything else runs in the library's kernels on the
shard's own tokens; the result is identical to one call over the whole group.

`all_gather` is any function mapping a per-shard tensor to the stacked tensor
of all shards ([S, ...], shard order): torch.distributed over NCCL across
GPUs, or a plain stack when the shards are run one after another in one
process.
"""
import torch

from . import native as nat


def dist_all_gather(group=None):
    """all_gather over torch.distributed, stacked in rank order."""
    import torch.distributed as dist

    def gather(t):
        parts = [torch.empty_like(t) for _ in range(dist.get_world_size(group))]
        dist.all_gather(parts, t.contiguous(), group=group)
        return torch.stack(parts)
    return gather


class Shard:
    """Buffers and calls of one shard (T_shard tokens) of a routing group whose
    capacity is C_group."""

    def __init__(self, T_shard, d_model, d_ff, n_experts, top_k, C_group, dtype, act, weights, alpha=1e-2,
                 device="cuda"):
        self.cfg = nat.config(T_shard, d_model, d_ff, n_experts, top_k, C_group, dtype, act, alpha)
        self.w = weights                           # device tensors, keys w_r b_r w1 b1 w3 b3 w2 b2
        self.ws = nat.new_workspace(self.cfg, device)
        T, k, N, d = T_shard, top_k, n_experts, d_model
        R = max(1, min(k * T, N * C_group))
        act_t = torch.bfloat16 if dtype == "bf16" else torch.float32
        i32, f32, f64 = torch.int32, torch.float32, torch.float64
        self.T, self.N, self.k, self.alpha = T, N, k, alpha
        self.idx = torch.empty(T, k, dtype=i32, device=device)
        self.gate = torch.empty(T, k, dtype=f32, device=device)
        self.pos = torch.empty(T, k, dtype=i32, device=device)
        self.drop = torch.empty(T, k, dtype=torch.uint8, device=device)
        self.counts = torch.empty(k, N, dtype=i32, device=device)
        self.claims = torch.empty(k, N, dtype=i32, device=device)
        self.claim_base = torch.empty(k, N, dtype=i32, device=device)
        self.kept = torch.empty(N, dtype=i32, device=device)
        self.offsets = torch.empty(N + 1, dtype=i32, device=device)
        self.row_token = torch.empty(R, dtype=i32, device=device)
        self.row_gate = torch.empty(R, dtype=f32, device=device)
        self.xe = torch.empty(R, d, dtype=act_t, device=device)
        self.ye = torch.empty(R, d, dtype=act_t, device=device)
        self.out = torch.empty(T, d, dtype=act_t, device=device)
        self.f = torch.empty(N, dtype=f64, device=device)
        self.P = torch.empty(N, dtype=f64, device=device)
        self.aux_local = torch.empty(1, dtype=f64, device=device)
        self.tokens = torch.full((1,), T, dtype=torch.int64, device=device)

    def route_and_count(self, x):
        w = self.w
        nat.check(nat.moe_route(self.cfg, x, w["w_r"], w["b_r"], self.idx, self.gate, None, self.f, self.P,
                                self.aux_local, self.ws))
        nat.check(nat.moe_expert_counts(self.cfg, self.idx, self.claims))
        return self.claims

    def dispatch(self, x, all_claims, shard):
        nat.check(nat.moe_claim_base(all_claims, all_claims.shape[0], shard, self.k, self.N, self.claim_base))
        nat.check(nat.moe_dispatch_shard(self.cfg, x, self.idx, self.gate, self.claim_base, self.pos, self.drop,
                                         self.counts, self.kept, self.offsets, self.row_token, self.row_gate,
                                         self.xe, self.ws))

    def experts_and_combine(self):
        w = self.w
        nat.check(nat.moe_expert_ffn(self.cfg, self.xe, self.offsets, w["w1"], w["b1"], w["w3"], w["b3"],
                                     w["w2"], w["b2"], self.ye, self.ws))
        nat.check(nat.moe_combine_shard(self.cfg, self.ye, self.idx, self.pos, self.drop, self.gate,
                                        self.offsets, self.claim_base, self.counts, self.out))
        return self.out

    def group_aux(self, all_tokens, all_f, all_P, f, P, aux):
        nat.check(nat.moe_aux_shards(all_tokens.shape[0], self.N, all_tokens, all_f, all_P, self.alpha, f, P, aux))


def sharded_forward(shards, xs, all_gather, first_index=0, mark=None):
    """Run the forward of the given shards (shards[i] on input xs[i], group
    shard index first_index + i) with the exchanges done by all_gather.  In one
    process (emulation) pass every shard with local_stack; across GPUs each rank
    passes its own shard, first_index = rank, and rank_all_gather.  mark
    (optional) is called with "experts" and "experts_done" around the expert
    FFN and combine calls (e.g. to record CUDA events there).
    Returns (outputs, group f, group P, group aux) of the shards given."""
    claims = [s.route_and_count(x) for s, x in zip(shards, xs)]
    all_claims = all_gather(claims)
    for i, (s, x) in enumerate(zip(shards, xs)):
        s.dispatch(x, all_claims, first_index + i)
    if mark:
        mark("experts")
    outs = [s.experts_and_combine() for s in shards]
    if mark:
        mark("experts_done")
    all_tokens = all_gather([s.tokens for s in shards]).reshape(-1)
    all_f = all_gather([s.f for s in shards])
    all_P = all_gather([s.P for s in shards])
    ref = shards[0]
    f = torch.empty_like(ref.f)
    P = torch.empty_like(ref.P)
    aux = torch.empty(1, dtype=torch.float64, device=ref.f.device)
    ref.group_aux(all_tokens, all_f.reshape(-1, ref.N), all_P.reshape(-1, ref.N), f, P, aux)
    return outs, f, P, aux


def local_stack(tensors):
    """all_gather for shards run one after another in one process."""
    return torch.stack(list(tensors))


def rank_all_gather(group=None):
    """all_gather for one shard per rank: takes the rank's one-element list."""
    g = dist_all_gather(group)
    return lambda tensors: g(tensors[0])
