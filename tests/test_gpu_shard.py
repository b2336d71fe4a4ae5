"""One routing group split into contiguous shards, run one after another on one
GPU (the exchange is a stack of the shards' count tables): routing integers
and outputs must be identical to a single call over the whole group, and the
group's f, P and aux loss must match it (f exactly, P and aux to fp32
summation error).  Needs a B200."""
import numpy as np
import pytest

import oracle
from gpu_helpers import REL_PROB, assert_close_out, oracle_layer
from mixture_experts_sparse_b200 import inputs
from mixture_experts_sparse_b200 import native as nat
from mixture_experts_sparse_b200.layer import MoeLayer, to_device, to_host_bits
from mixture_experts_sparse_b200.shard import Shard, local_stack, sharded_forward

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)


def _split_api_full(L, T, d, dff, N, k, C, dtype, act):
    """The whole group through the split entry points (route, dispatch, experts,
    combine): the same arithmetic path the shards take."""
    s = Shard(T, d, dff, N, k, C, dtype, act, {key: to_device(L.get(key)) for key in
                                                 ("w_r", "b_r", "w1", "b1", "w3", "b3", "w2", "b2")})
    x = to_device(L["x"])
    outs, f, P, aux = sharded_forward([s], [x], local_stack)
    torch.cuda.synchronize()
    return s, outs[0], aux


@pytest.mark.parametrize("k,act,dtype,cf", [(1, "relu", "bf16", 1.0), (2, "relu", "bf16", 1.0),
                                             (2, "swiglu", "bf16", 1.25), (1, "relu", "f32", 1.0)])
def test_three_shards_equal_one_group(k, act, dtype, cf):
    T, d, dff, N = 5000, 128, 256, 8
    bounds = [0, 1700, 3300, T]          # uneven contiguous shards
    L = inputs.make_layer(T=T, d_model=d, d_ff=dff, n_experts=N, top_k=k, act=act, dtype=dtype, seed=77 + k,
                          biases=(dtype == "f32"), router_bias=np.linspace(0.4, 0.0, N).astype(np.float32))
    C = nat.moe_capacity(T, N, k, cf)
    W = {key: to_device(L.get(key)) for key in ("w_r", "b_r", "w1", "b1", "w3", "b3", "w2", "b2")}
    shards, xs = [], []
    for a, b in zip(bounds[:-1], bounds[1:]):
        shards.append(Shard(b - a, d, dff, N, k, C, dtype, act, W))
        xs.append(to_device(L["x"][a:b]))
    outs, f, P, aux = sharded_forward(shards, xs, local_stack)
    torch.cuda.synchronize()
    for s in shards:
        nat.check(nat.moe_read_device_status(s.ws))

    full, full_out, full_aux = _split_api_full(L, T, d, dff, N, k, C, dtype, act)
    cat = lambda name: np.concatenate([getattr(s, name).cpu().numpy() for s in shards])
    np.testing.assert_array_equal(cat("idx"), full.idx.cpu().numpy())
    np.testing.assert_array_equal(cat("pos"), full.pos.cpu().numpy())      # group-wide claim numbers
    np.testing.assert_array_equal(cat("drop"), full.drop.cpu().numpy())
    np.testing.assert_array_equal(sum(s.kept.cpu().numpy() for s in shards), full.kept.cpu().numpy())
    got = np.concatenate([to_host_bits(o) for o in outs])
    np.testing.assert_array_equal(got, to_host_bits(full_out))           # bit-identical outputs
    # f is a ratio of integer counts; P and aux come from fp32 per-tile partial
    # sums of the probabilities, whose tiles differ between the shards and the
    # single call, so they agree to fp32 summation error, not bitwise
    np.testing.assert_allclose(f.cpu().numpy(), full.f.cpu().numpy(), rtol=1e-14, atol=0)
    np.testing.assert_allclose(P.cpu().numpy(), full.P.cpu().numpy(), rtol=REL_PROB, atol=0)
    assert abs(aux.item() - full_aux.item()) <= REL_PROB * abs(full_aux.item())
    # and the group matches the oracle
    res = oracle_layer(L, k, C, act, dtype)
    np.testing.assert_array_equal(cat("pos"), res["disp"]["pos"])
    assert_close_out(oracle.widen(got) if dtype == "bf16" else got.astype(np.float64), res["out_exact"], dtype)
    np.testing.assert_allclose(f.cpu().numpy(), res["f"], rtol=1e-14, atol=0)
    assert abs(aux.item() - res["aux"]) <= REL_PROB * abs(res["aux"])


def test_claim_base_rule():
    # shards' counts [S, k, N]; base[0] = earlier shards' rank-0 claims,
    # base[1] = all rank-0 claims + earlier shards' rank-1 claims
    S, k, N = 3, 2, 5
    rng = np.random.default_rng(0)
    cnt = rng.integers(0, 50, size=(S, k, N)).astype(np.int32)
    dev = torch.from_numpy(cnt).cuda()
    for s in range(S):
        base = torch.empty(k, N, dtype=torch.int32, device="cuda")
        nat.check(nat.moe_claim_base(dev, S, s, k, N, base))
        want0 = cnt[:s, 0].sum(0)
        want1 = cnt[:, 0].sum(0) + cnt[:s, 1].sum(0)
        np.testing.assert_array_equal(base.cpu().numpy(), np.stack([want0, want1]))
