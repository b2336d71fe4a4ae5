"""Parity of the persistent grouped GEMM's multi-tile path with the CPU oracle,
on every token.  Needs a B200.

The small full-oracle layers of test_gpu_parity.py have fewer tiles than the
GPU has CTA pairs, so every CTA runs at most one tile there.  These mid-size
layers give each CTA pair at least three tiles in both expert GEMMs (asserted
from the oracle's kept counts), so they run the persistent loop's later
tiles, the swap between the two TMEM accumulators and the shared-memory ring
wrapping across tiles -- and the oracle still evaluates every token (its
per-token work is spread over the host's threads).  Each layer is checked
with the CTA-pair kernels (the default) and with the one-CTA kernels
(MOE_B200_GEMM=single, in a subprocess: the choice is read at library load).
"""
import os
import subprocess
import sys

import pytest

from gpu_helpers import assert_close_out, compare_routing, host_threads, oracle_layer_threads, run_layer, widen_out
from mixture_experts_sparse_b200 import inputs
from mixture_experts_sparse_b200 import native as nat

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

# T, d, d_ff, N, k, cf, act
MID = [
    (32768, 512, 1024, 16, 1, 1.25, "relu"),
    (16384, 512, 1024, 16, 2, 1.25, "swiglu"),
]


def _tiles(kept, rows_per_tile, n_dim, cols_per_tile):
    mt = sum(-(-int(v) // rows_per_tile) for v in kept)
    return mt * -(-n_dim // cols_per_tile)


def _check_mid(case, pair):
    T, d, dff, N, k, cf, act = case
    C = nat.moe_capacity(T, N, k, cf)
    L = inputs.make_layer(T=T, d_model=d, d_ff=dff, n_experts=N, top_k=k, act=act, dtype="bf16", seed=T + k)
    res = oracle_layer_threads(L, k, C, act, "bf16")
    kept = res["disp"]["kept"]
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    ctas = sms // 2 if pair else sms
    rows = 256 if pair else 128
    bn1 = 128 if act == "swiglu" else 256
    t1 = _tiles(kept, rows, dff, bn1)
    t2 = _tiles(kept, rows, d, 256)
    assert t1 >= 3 * ctas and t2 >= 3 * ctas, (t1, t2, ctas)
    layer, _ = run_layer(L, T, d, dff, N, k, C, "bf16", act)
    compare_routing(layer, res)
    assert_close_out(widen_out(layer.out), res["out_exact"], "bf16")
    return t1, t2, ctas


@pytest.mark.parametrize("case", MID, ids=lambda c: "T{}_d{}_ff{}_N{}_k{}_{}".format(*c[:5], c[6]))
def test_mid_size_every_token_pair_kernels(case):
    t1, t2, ctas = _check_mid(case, pair=True)
    print(f"\ntiles: stage 1 {t1}, stage 2 {t2} over {ctas} CTA pairs; oracle on {host_threads()} host threads")


def test_mid_size_every_token_single_cta_kernels():
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    code = (
        "import sys; sys.path.insert(0, %r); sys.path.insert(0, %r)\n"
        "from test_gpu_persistent_gemm import MID, _check_mid\n"
        "for case in MID:\n"
        "    _check_mid(case, pair=False)\n"
        "print('single ok')\n" % (root, os.path.join(root, "tests")))
    env = dict(os.environ, MOE_B200_GEMM="single")
    r = subprocess.run([sys.executable, "-c", code], env=env, capture_output=True, text=True, timeout=900)
    assert r.returncode == 0 and "single ok" in r.stdout, r.stdout[-2000:] + r.stderr[-4000:]
