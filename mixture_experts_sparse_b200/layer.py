"""Device-side buffers for one MoE layer, driven through the C ABI.

PyTorch only provides device memory and streams here; every step of the layer
runs in libmoe_b200's kernels (see ``native``).
"""
import numpy as np

from . import native as nat

WEIGHT_KEYS = ("w_r", "b_r", "w1", "b1", "w3", "b3", "w2", "b2")


def to_device(a, device="cuda"):
    """numpy -> torch on `device`; uint16 arrays are bf16 bit patterns."""
    import torch
    if a is None:
        return None
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16)).to(device).view(torch.bfloat16)
    return torch.from_numpy(a).to(device)


def to_host_bits(t):
    """torch bf16 tensor -> numpy uint16 bit patterns; other dtypes -> numpy."""
    import torch
    t = t.detach().cpu()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.numpy()


class MoeLayer:
    """Weights, workspace and routing outputs of one layer on one GPU."""

    def __init__(self, T, d_model, d_ff, n_experts, top_k, capacity, dtype, act, weights, alpha=1e-2,
                 device="cuda", priority=False):
        import torch
        self.cfg = nat.config(T, d_model, d_ff, n_experts, top_k, capacity, dtype, act, alpha, priority=priority)
        self.device = device
        self.w = {k: to_device(weights.get(k), device) for k in WEIGHT_KEYS}
        self.ws = nat.new_workspace(self.cfg, device)
        self.act_dtype = torch.bfloat16 if dtype == "bf16" else torch.float32
        i32, f32, f64 = torch.int32, torch.float32, torch.float64
        k, N = top_k, n_experts
        self.out = torch.empty(T, d_model, dtype=self.act_dtype, device=device)
        self.idx = torch.empty(T, k, dtype=i32, device=device)
        self.gate = torch.empty(T, k, dtype=f32, device=device)
        self.pos = torch.empty(T, k, dtype=i32, device=device)
        self.drop = torch.empty(T, k, dtype=torch.uint8, device=device)
        self.counts = torch.empty(k, N, dtype=i32, device=device)
        self.kept = torch.empty(N, dtype=i32, device=device)
        self.offsets = torch.empty(N + 1, dtype=i32, device=device)
        self.f = torch.empty(N, dtype=f64, device=device)
        self.P = torch.empty(N, dtype=f64, device=device)
        self.aux = torch.empty(1, dtype=f64, device=device)

    def forward(self, x, stream=None, routing_outputs=True):
        """One layer forward on device input x; returns the status code."""
        w = self.w
        r = routing_outputs
        return nat.moe_forward(self.cfg, x, w["w_r"], w["b_r"], w["w1"], w["b1"], w["w3"], w["b3"], w["w2"],
                               w["b2"], self.out,
                               self.idx if r else None, self.gate if r else None, self.pos if r else None,
                               self.drop if r else None, self.counts if r else None, self.kept if r else None,
                               self.offsets if r else None, self.f if r else None, self.P if r else None,
                               self.aux, ws=self.ws, stream=stream)
