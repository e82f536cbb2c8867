"""GPU parity of the grouped decode call (rabit_gemv_grouped) against the float64 oracle.

One launch computes several independent layers; every layer's output must meet the bar of
rabit_gemv (normwise <= 2e-3 for bf16 x, <= 1e-5 for fp32 x), and so must rabit_gemv on the
same layer alone.  The two need not agree bit for bit: the share of each CTA, and with it the
runs of columns that share one z scale, depends on all the work in the launch.
"""
import numpy as np
import pytest
import torch

import oracle
from bit_gemv_rabit_b200 import inputs
from bit_gemv_rabit_b200 import rabit

pytestmark = pytest.mark.gpu

TOL = {torch.bfloat16: 2e-3, torch.float32: 1e-5}


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    from bit_gemv_rabit_b200 import build
    build.build()
    oracle.build()
    rabit.load()
    yield
    assert rabit.rabit_read_fault(clear=True) == 0


def normwise(y, ref):
    return float(np.max(np.abs(y - ref)) / max(np.max(np.abs(ref)), 1e-300))


def _layer(seed, N, K, batch, xdtype, P=2, outliers=0.0):
    W = inputs.weight(seed, N, K, outlier_frac=outliers)
    a, b = inputs.scales(seed, W, P=P)
    x = inputs.activations(seed + 1, batch, K)                      # bf16 bits
    at, bt = torch.from_numpy(a).cuda(), torch.from_numpy(b).cuda()
    packed = rabit.alloc_packed(N, K, P=P)
    rabit.rabit_derive_pack(torch.from_numpy(W).cuda(), at, bt, packed, P=P)
    xt = torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).cuda()
    if xdtype == torch.float32:
        xt = xt.float()
        xh = inputs.bf16_to_f32(x)
    else:
        xh = x
    S = oracle.derive_signs(W, a, b, P=P)
    y = torch.full((batch, N), float("nan"), device="cuda")
    return dict(packed=packed, a=at, b=bt, N=N, K=K, x=xt, y=y, ref=oracle.layer(S, a, b, xh))


@pytest.mark.parametrize("xdtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("batch", [1, 3, 9])
def test_grouped_layers_match_oracle_and_single_calls(xdtype, batch):
    # mixed shapes: ragged rows and columns, a layer smaller than one tile, one larger
    shapes = [(300, 1000), (4096, 520), (77, 4096), (1024, 2048)]
    layers = [_layer(7000 + i, N, K, batch, xdtype, outliers=0.001) for i, (N, K) in enumerate(shapes)]
    rabit.rabit_gemv_grouped([(L["packed"], L["a"], L["b"], L["N"], L["K"], L["x"], L["y"]) for L in layers])
    torch.cuda.synchronize()
    for L in layers:
        y = L["y"].cpu().numpy().astype(np.float64)
        err = normwise(y, L["ref"])
        assert err <= TOL[xdtype], (L["N"], L["K"], err)
        alone = torch.empty_like(L["y"])
        rabit.rabit_gemv(L["packed"], L["a"], L["b"], L["N"], L["K"], L["x"], alone)
        torch.cuda.synchronize()
        assert normwise(alone.cpu().numpy().astype(np.float64), L["ref"]) <= TOL[xdtype], (L["N"], L["K"])


def test_grouped_three_paths():
    layers = [_layer(7100 + i, N, K, 2, torch.bfloat16, P=3) for i, (N, K) in enumerate([(500, 700), (256, 4096)])]
    rabit.rabit_gemv_grouped([(L["packed"], L["a"], L["b"], L["N"], L["K"], L["x"], L["y"]) for L in layers], P=3)
    torch.cuda.synchronize()
    for L in layers:
        assert normwise(L["y"].cpu().numpy().astype(np.float64), L["ref"]) <= 2e-3


def test_grouped_llama2_7b_decode_set_one_launch():
    """The seven projection shapes of the Llama-2-7B decode set in one launch, batch 1, every
    output row checked against the oracle."""
    spec = inputs.WORKLOADS["llama2_7b_decode_b1"]
    layers = []
    for idx, (name, N, K) in enumerate(spec["set"]):
        seed = inputs.seed_for(spec["cfg"], idx)
        W = inputs.weight(seed, N, K, sigma=spec["sigma"])
        a, b = inputs.scales(seed, W)
        x = inputs.activations(seed, 1, K)
        at, bt = torch.from_numpy(a).cuda(), torch.from_numpy(b).cuda()
        packed = rabit.alloc_packed(N, K)
        rabit.rabit_derive_pack(torch.from_numpy(W).cuda(), at, bt, packed)
        S = oracle.derive_signs(W, a, b)
        layers.append(dict(packed=packed, a=at, b=bt, N=N, K=K,
                           x=torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).cuda(),
                           y=torch.full((1, N), float("nan"), device="cuda"), ref=oracle.layer(S, a, b, x)))
        del W
    ws = rabit.alloc_gemv_grouped_workspace([(L["packed"], L["a"], L["b"], L["N"], L["K"], L["x"], L["y"])
                                             for L in layers])
    for _ in range(2):   # the workspace's counters are left at zero for the next call
        rabit.rabit_gemv_grouped([(L["packed"], L["a"], L["b"], L["N"], L["K"], L["x"], L["y"]) for L in layers],
                                 workspace=ws)
        torch.cuda.synchronize()
        for L in layers:
            assert normwise(L["y"].cpu().numpy().astype(np.float64), L["ref"]) <= 2e-3


def test_prepared_group_matches_the_plain_call_as_x_changes():
    """GemvGroup marshals the call once; each run reads the tensors' current contents, so new
    x (written in place, as an end-to-end step does) gives the plain call's y bit for bit,
    and y meets the oracle's bar.  x and y are views of one flat buffer each."""
    shapes = [(4096, 4096), (1024, 4096), (512, 11008)]
    layers = [_layer(7300 + i, N, K, 1, torch.bfloat16) for i, (N, K) in enumerate(shapes)]
    xflat = torch.empty(sum(K for _, K in shapes), dtype=torch.bfloat16, device="cuda")
    yflat = torch.empty(sum(N for N, _ in shapes), dtype=torch.float32, device="cuda")
    tup, xo, yo = [], 0, 0
    for L in layers:
        tup.append((L["packed"], L["a"], L["b"], L["N"], L["K"], xflat[xo:xo + L["K"]].view(1, L["K"]),
                    yflat[yo:yo + L["N"]].view(1, L["N"])))
        xo += L["K"]
        yo += L["N"]
    group = rabit.GemvGroup(tup)
    for step in range(2):
        xs = [inputs.activations(7400 + 10 * step + i, 1, K) for i, (_, K) in enumerate(shapes)]
        xflat.copy_(torch.from_numpy(np.concatenate([x.view(np.int16).reshape(-1) for x in xs]))
                    .view(torch.bfloat16))
        group.run()
        got = yflat.clone()
        yflat.fill_(float("nan"))
        rabit.rabit_gemv_grouped(tup, workspace=group.workspace)
        torch.cuda.synchronize()
        assert torch.equal(got, yflat)
        yo = 0
        for i, (x, (N, K)) in enumerate(zip(xs, shapes)):
            W = inputs.weight(7300 + i, N, K)
            a, b = inputs.scales(7300 + i, W)
            ref = oracle.layer(oracle.derive_signs(W, a, b), a, b, x)
            assert normwise(got[yo:yo + N].cpu().numpy()[None, :], ref) <= TOL[torch.bfloat16]
            yo += N
